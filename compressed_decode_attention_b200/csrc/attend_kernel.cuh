// tq_attend: decode attention over the packed cache in one persistent,
// load-balanced kernel on the B200 tensor cores.
//
// [ADAPTQ §How it works, item 3]: the query is rotated once; scores are
// formed from the packed indices through the codebook, without materializing
// the dequantized cache. [TQAI §Test Suite]: the target is
// softmax(Q·K^T/sqrt d)·V. [TQPLUS §2 Sparse V]: V rows with negligible
// weight are left out (block-local rule, include/tq.h).
//
// Head dimension D = 64, 128 or 256 is a template parameter: d/32 query and
// output values per lane, d/16 k-steps per score MMA chain and d/16 PV
// coordinate tiles.
//
// Work decomposition. The cache is a list of (batch, kv head) segments of
// 64-position blocks. Each segment costs its blocks plus a fixed overhead
// (kSegCost block units: query rotation, first-chunk latency, merges), and
// CTA c of Geff owns the blocks in the cost range [c·C/Geff, (c+1)·C/Geff)
// of the total cost C, so CTAs whose range holds many short segments get
// fewer blocks. Geff = min(grid, #blocks), except that when all S segments
// have the same block count and S <= grid, Geff is the largest multiple of
// S within the grid (at most one CTA per block) and the overhead is 0, so
// every CTA stays inside one segment. A CTA walks the segments of its
// range. Its warps split each segment in whole units, merge in shared
// memory, and either write the output (segment = whole sequence) or leave a
// partial in a workspace slot; the last CTA to finish a sequence (atomic
// counter, no waiting) merges the partials and writes the output. No
// separate combine launch, no spin-waits on other CTAs.
//
// Per warp and chunk of up to 64 positions (GQA group of g <= 8 query heads),
// in four 16-position steps:
//   stage   bulk copies (cp.async.bulk, one lane) of the packed K/V rows and
//           fp16 norms into a per-warp ring of shared-memory slots, each
//           completed on its own mbarrier (bounded wait)
//   scores  mma.m16n8k16, fp16 in, fp32 accumulate, per 8 positions: A rows
//           0-7 = K codebook high parts, rows 8-15 = low parts of the same
//           positions (one shared-table entry per packed byte fills two
//           fragment registers); B = rotated query, fp16 high and low parts
//           in the 8 columns (g <= 4: 4 heads x {high, low}; g <= 8: two
//           column tiles). K high, K low and query low are summed, so scores
//           keep ~22 significant bits (fp16-only operands measured up to
//           1.2e-2 output error with x20 outlier channels).
//   softmax fp32, log2 domain; chunk maximum = sparse-V block maximum.
//   PV      mma.m16n8k16: A = V codebook values (fp16), coordinates x
//           positions; B = softmax weight x V norm (fp16), moved from the
//           score layout with movmatrix. V2: position pairs by byte permutes
//           of a 4-entry register table; V3/V4: pair table + movmatrix.
// Output, once per (batch, query head): D⊙(H·(acc/l))/d with shuffles.
#pragma once
#include <atomic>
#include <math.h>

#include <type_traits>

#include "encode_common.cuh"

namespace tq {
namespace {

// Warps per CTA: 12, or 8 at d = 256 where a 64-position stage of the K and
// V rows is twice as large.

constexpr int kMaxWarps = 12;
constexpr int kBlk = kGateBlock;                // positions per block
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kKScale = 256.f;                // K codebook scale inside the MMA
// Shared memory of one CTA when `per_sm` CTAs share an SM's 228 KB (1 KB of
// each CTA's share is reserved by the system).
constexpr int smem_budget(int per_sm) { return per_sm == 1 ? 227 * 1024 : 228 * 1024 / per_sm - 1024; }
constexpr int kMaxStages = 3;                   // ring slots per warp
#ifdef TQ_TEST_INJECT_WAIT_FAULTS
// Test build only (libtq_waittest.so, for the test of the give-up path):
// waits give up after ~50 us, and two waits are made to run out without any
// invalid access: in tq_attend, every warp arms the ring slot of its first
// chunk for 16 bytes more than its bulk copies deliver (all their bytes
// still land, so nothing is in flight when it stops), and in the decode step
// the helper warp never raises the flag its owner waits for.
constexpr long long kWaitLimitCycles = 100000LL;
constexpr bool kInjectWaitFaults = true;
#else
// Give up on a staged-data wait after this many cycles (~1 s at 2 GHz).
constexpr long long kWaitLimitCycles = 2000000000LL;
constexpr bool kInjectWaitFaults = false;
#endif

constexpr int ceil_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// misc words
constexpr int kMiscCost = 0;     // total cost (lo, hi), per-segment overhead sig
constexpr int kMiscDesc = 48;    // segment: b, g, blk0, nseg, nb, L, cost of block 0 (lo, hi)
// Cost of one (sequence, kv head) segment in the CTA split, in 64-position
// block units, on top of its blocks: the query rotation, the first chunk's
// latency, the merges and the share of a last round of blocks.
constexpr int kSegCost = 16;
constexpr int kMiscLast = 8;     // last-CTA flag
constexpr int kMiscNB = 9;       // flat block count (lo, hi), common length
constexpr int kMiscState = 12;   // scan state: sb, sP (lo, hi)
constexpr int kMiscQInv = 16;    // 8 floats: 1/(query scale · kKScale)
constexpr int kMiscApp = 24;     // decode-step append: segment count + 1 once encoded
constexpr int kMiscM = 32;       // 8 floats: merged max
constexpr int kMiscL = 40;       // 8 floats: merged sum
constexpr int kMiscCb = 64;      // 32 words: staged codebooks
constexpr int kMiscWt = 128;     // warps x 8 floats: per-warp merge weights
constexpr int kMiscWords = 256;  // Geo::MISC / 4
static_assert(kMiscWt + kMaxWarps * kMaxGroup <= kMiscWords, "misc words");

// Sizes that follow the head dimension D.
template <int D>
struct Dm {
  static constexpr int QPL = D / 32;          // query / output values per lane
  static constexpr int KS = D / 16;           // k-steps of the score MMA
  static constexpr int NPV = D / 16;          // coordinate tiles of the PV MMA
  static constexpr float ROOT = D == 64 ? 8.f : D == 128 ? 11.3137084989847603904f : 16.f;
  // Per-warp merge buffer (floats): accumulators (in register order, D/4 per
  // lane at a stride of LANE, which keeps 16-byte stores of consecutive lanes
  // on distinct banks; or in output order), then per-head max and sum.
  static constexpr int LANE = D / 4 + 4;
  static constexpr int M = 32 * LANE;
  static constexpr int L = M + kMaxGroup;
  static constexpr int STRIDE = L + kMaxGroup;
  static_assert(M >= kMaxGroup * D, "merge buffer holds GQ x D outputs");
};

template <int BK, int BV, int D, bool WIDE>
struct GeoL {
  static constexpr int RK = D * BK / 8;                 // packed K row bytes
  static constexpr int RV = D * BV / 8;
  // rows per 16-byte multiple of a bulk copy of K / V rows
  static constexpr int KROWS = RK % 16 == 0 ? 1 : 16 / (RK % 16);
  static constexpr int VROWS = RV % 16 == 0 ? 1 : 16 / (RV % 16);
  static_assert((KROWS * RK) % 16 == 0 && (VROWS * RV) % 16 == 0, "row multiple");
  static_assert(kGateBlock % KROWS == 0 && kGateBlock % VROWS == 0 && 8 % KROWS == 0 &&
                8 % VROWS == 0, "rounded row counts stay inside a block and cap_tok");
  static constexpr int RVS = RV;                        // V row stride in smem
  static constexpr int KB = kBlk * RK;
  static constexpr int VB = kBlk * RVS;
  static constexpr int NKOFF = KB + VB;
  static constexpr int STAGE = KB + VB + 2 * kBlk * 2;
  // K table: uint2 (high pair, low pair) per (pair code, lane & 15): 128 B per
  // code. In the wide layout (4-bit K: the pair code is a whole byte) codes
  // are 256 B apart, so that one byte permute of the packed word and the
  // lane offset forms the entry's address; the V table (3/4 bits) then sits
  // in the other 128 B of each code's row.
  static constexpr bool KWIDE = WIDE;
  static constexpr int KSTRIDE = WIDE ? 256 : 128;
  static constexpr int LUTK = (1 << (2 * BK)) * KSTRIDE;
  // V table (3/4 bits): uint32 fp16 pair per (pair code, lane): 128 B per code.
  static constexpr int LUTV = BV == 2 || WIDE ? 0 : (1 << (2 * BV)) * 128;
  // Narrow layout: the V table sits at a power-of-two offset no smaller
  // than either table, so entry addresses are formed with OR.
  static constexpr int LUTV_OFF = WIDE ? 128 : BV == 2 ? LUTK : ceil_pow2(LUTK > LUTV ? LUTK : LUTV);
  static constexpr int VSHIFT = WIDE ? 8 : 7;           // log2 of the V code stride
  static constexpr int QOFF = WIDE ? LUTK : LUTV_OFF + LUTV;
  static constexpr int QS = kMaxGroup * D * 2 * 2;      // q~ high and low, fp16
  static constexpr int MISC = 1024;                     // kMiscWords words
  static constexpr int MBAR = kMaxWarps * kMaxStages * 8;  // per-warp ring barriers
  static constexpr int APPOFF = QOFF + QS + MISC + MBAR;  // decode-step append:
  static constexpr int APP = D + 64;                    //   K row, V row, norms
  static constexpr int FIXED = APPOFF + APP;
  // One CTA of 12 warps per SM (8 at d = 256, where a stage of K/V rows is
  // twice as large). Measured: two 6-warp CTAs per SM (halved shared memory)
  // made the attention launch 9% slower on the Llama-3-8B-shaped layer.
  static constexpr int PER_SM = 1;
  static constexpr int NW = D == 256 ? 8 : 12;
  static constexpr int BUDGET = smem_budget(PER_SM);
  static constexpr int NFIT = (BUDGET - FIXED) / (NW * STAGE);
  static constexpr int NSTAGE = NFIT > kMaxStages ? kMaxStages : NFIT;
  static constexpr int MERGE = NW * Dm<D>::STRIDE * 4;
  static constexpr int RING = NSTAGE * NW * STAGE;
  static constexpr int SMEM = FIXED + (RING > MERGE ? RING : MERGE);
  static_assert(NSTAGE >= 1 || WIDE, "stage ring does not fit");
  static_assert(SMEM <= BUDGET || WIDE, "shared memory budget");
};

// The wide K table wherever it keeps the ring as deep as the narrow one.
template <int BK, int BV, int D>
struct Geo : GeoL<BK, BV, D, (BK == 4 && GeoL<BK, BV, D, true>::NSTAGE >= 1 &&
                              GeoL<BK, BV, D, true>::NSTAGE >= GeoL<BK, BV, D, false>::NSTAGE)> {
  static_assert(!Geo::KWIDE || (BK == 4 && BV <= BK), "wide layout: byte pair codes, V codes fit");
};


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

// Shared-memory barrier with a transaction count, completed by bulk copies.
__device__ __forceinline__ void mbar_init(uint32_t bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done) : "r"(bar), "r"(parity) : "memory");
  return done != 0;
}
// Slow path of mbar_wait, out of line: keeps polling until the phase
// completes or kWaitLimitCycles have passed.
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try(bar, parity))
    if (clock64() - t0 > kWaitLimitCycles) return false;
  return true;
}
// Waits (bounded, out of line) until the shared word at `flag` equals
// `want`; false if it does not within kWaitLimitCycles.
__device__ __noinline__ bool wait_flag_slow(const int* flag, int want) {
  const long long t0 = clock64();
  while (*reinterpret_cast<const volatile int*>(flag) != want) {
    if (clock64() - t0 > kWaitLimitCycles) return false;
    __nanosleep(64);
  }
  return true;
}
// Waits for the phase with the given parity to complete; false if it does
// not within kWaitLimitCycles.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  return mbar_try(bar, parity) || mbar_wait_slow(bar, parity);
}
// Bulk copy global -> this CTA's shared memory (16-byte aligned, size a
// multiple of 16), completing on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

template <typename T>
__device__ __forceinline__ T lds(const uint8_t* base, uint32_t off) {
  return *reinterpret_cast<const T*>(base + off);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ int seq_blocks(const AttendArgs& a, int b) {
  const int L = min(max(a.ctx_lens[b], 0), a.cap_tok);
  return (L + kBlk - 1) / kBlk;
}

// CTA owning the block at cost `blk` when a total cost NB is split over G
// CTAs as [c·NB/G, (c+1)·NB/G): the largest c with floor(c·NB/G) <= blk.
__device__ __forceinline__ int cta_of(long long blk, long long nb, int g) {
  return (int)(((blk + 1) * g - 1) / nb);
}

// Walsh-Hadamard transform of 32·Q values spread as Q per lane (coordinate
// Q·lane + k in x[k]): log2(Q) in-register stages, five shuffle stages.
template <int Q>
__device__ __forceinline__ void fwht_warp(float (&x)[Q], int lane) {
#pragma unroll
  for (int s = 1; s < Q; s <<= 1)
#pragma unroll
    for (int k = 0; k < Q; ++k)
      if (!(k & s)) {
        const float u = x[k], v = x[k + s];
        x[k] = u + v;
        x[k + s] = u - v;
      }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const bool upper = lane & o;
#pragma unroll
    for (int k = 0; k < Q; ++k) {
      const float p = __shfl_xor_sync(0xFFFFFFFFu, x[k], o);
      x[k] = upper ? p - x[k] : x[k] + p;
    }
  }
}

// Output coordinate held by accumulator register (m-tile r, m-slot m) of PV.
template <int BV, int D>
__device__ __forceinline__ int pv_coord(int r, int m) {
  if (BV == 2) return (D / 8) * (m & 7) + 2 * r + (m >> 3);
  return (D / 4) * ((m & 7) >> 1) + 4 * r + (m & 1) + 2 * (m >> 3);
}

// Position of output (head h, coordinate c) in a warp's accumulators as
// stored lane-major (register acc[r][k] of a lane at 4r + k):
// the inverse of pv_coord together with the head columns 2tq, 2tq + 1.
template <int BV, int D>
__device__ __forceinline__ int pv_slot(int c, int h) {
  int m, r;
  if (BV == 2) {
    m = c / (D / 8) + 8 * (c & 1);
    r = (c % (D / 8)) >> 1;
  } else {
    m = 2 * (c / (D / 4)) + (c & 1) + 8 * ((c >> 1) & 1);
    r = (c % (D / 4)) >> 2;
  }
  const int lane = 4 * (m & 7) + (h >> 1);
  return lane * Dm<D>::LANE + 4 * r + (h & 1) + 2 * (m >> 3);
}

// The CB bytes at shared offset `off` (a lane's chunk of a packed row) as
// little-endian words, followed by a zero word. Loads as wide as the
// chunk's size and alignment allow (CB = d·bits/32: 6 .. 32 bytes).
template <int CB>
__device__ __forceinline__ void load_chunk(const uint8_t* base, uint32_t off,
                                           uint32_t (&w)[(CB + 3) / 4 + 1]) {
  constexpr int NW = (CB + 3) / 4;
  if constexpr (CB % 16 == 0) {
#pragma unroll
    for (int i = 0; i < CB / 16; ++i) {
      const uint4 u = lds<uint4>(base, off + 16 * i);
      w[4 * i] = u.x; w[4 * i + 1] = u.y; w[4 * i + 2] = u.z; w[4 * i + 3] = u.w;
    }
  } else if constexpr (CB % 8 == 0) {
#pragma unroll
    for (int i = 0; i < CB / 8; ++i) {
      const uint2 u = lds<uint2>(base, off + 8 * i);
      w[2 * i] = u.x; w[2 * i + 1] = u.y;
    }
  } else if constexpr (CB % 4 == 0) {
#pragma unroll
    for (int i = 0; i < CB / 4; ++i) w[i] = lds<uint32_t>(base, off + 4 * i);
  } else {                                          // 6 bytes, 2-byte aligned
    static_assert(CB == 6, "chunk size");
    const uint32_t h0 = lds<uint16_t>(base, off), h1 = lds<uint16_t>(base, off + 2);
    w[0] = h0 | (h1 << 16);
    w[1] = lds<uint16_t>(base, off + 4);
  }
  w[NW] = 0;
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

// Byte offset of the K table entry for pair code p of a lane's chunk (entries
// 128 bytes apart). For 4-bit codes the pair code is a whole byte: one byte
// permute and one multiply-add; narrower codes straddle bytes.
template <int BK>
__device__ __forceinline__ uint32_t k_entry(const uint32_t* w, int p) {
  if constexpr (BK == 4)
    return (uint32_t)__byte_perm(w[p >> 2], 0u, 0x4440u | (uint32_t)(p & 3)) * 128u;
  else
    return pair_code_shifted<BK, 7>(w, p);
}

template <int BK, int BV, int NT, int D>
__global__ void __launch_bounds__(32 * Geo<BK, BV, D>::NW, Geo<BK, BV, D>::PER_SM)
attend_kernel(const __grid_constant__ AttendArgs a,
              const __grid_constant__ Codebook cbk,
              const __grid_constant__ Codebook cbv,
              const __grid_constant__ SignMask sm) {
  using Gm = Geo<BK, BV, D>;
  using Dd = Dm<D>;
  constexpr int kWarps = Gm::NW, kThreads = 32 * kWarps;
  constexpr int QPL = Dd::QPL, KS = Dd::KS, NPV = Dd::NPV;
  constexpr int CBK = D * BK / 32, CBV = D * BV / 32;   // chunk bytes per tq lane
  constexpr int NR = NT == 1 ? 1 : 2;       // score rows (positions) per lane and step
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* lutK = smem;                                   // offset 0
  uint8_t* lutV = smem + Gm::LUTV_OFF;
  __half* qhi = reinterpret_cast<__half*>(smem + Gm::QOFF);
  __half* qlo = qhi + kMaxGroup * D;
  float* fin = reinterpret_cast<float*>(qhi);             // reuses q~ after a segment
  int* misc = reinterpret_cast<int*>(smem + Gm::QOFF + Gm::QS);
  float* miscf = reinterpret_cast<float*>(misc);
  float* merge = reinterpret_cast<float*>(smem + Gm::FIXED);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // this warp's ring barriers: one per slot, phases counted over all blocks
  // the warp stages in this launch (jdone)
  const uint32_t wbar = smem_addr(smem) + Gm::QOFF + Gm::QS + Gm::MISC + warp * kMaxStages * 8;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < Gm::NSTAGE; ++s) mbar_init(wbar + 8 * s);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncwarp();
  int jdone = 0;
  bool stalled = false;                       // a staged-data wait gave up
  const int gq = lane >> 2, tq = lane & 3;
  const int H = a.n_kv_heads, GQ = a.gqa, B = a.batch;
  const int Gc = gridDim.x, cta = blockIdx.x;   // Gc <= kMaxCtas (host check)
  const uint32_t lbK = (lane & 15) * 8;                   // K table lane offset
  const uint32_t lbV = Gm::LUTV_OFF | (lane * 4);         // V table lane base

  // Launches that follow in the stream may start their own set-up now; they
  // wait for this grid before touching memory (programmatic dependent
  // launch; a no-op without it).
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  // ---- codebooks staged in misc (launch parameters only): fp16 high/low
  // parts of the scaled K levels and the fp16 V levels
  uint32_t* cbs = reinterpret_cast<uint32_t*>(misc) + kMiscCb;
  if (tid < 16) {
    const float c = cbk.centroid[tid] * kKScale;
    const __half h = __float2half_rn(c), l = __float2half_rn(c - __half2float(h));
    cbs[tid] = (uint32_t)__half_as_ushort(h) | ((uint32_t)__half_as_ushort(l) << 16);
    cbs[16 + tid] = __half_as_ushort(__float2half_rn(cbv.centroid[tid]));
  }
  __syncthreads();
  // ---- K table: uint2 (high pair, low pair) per (pair code, copy)
  for (int e = tid; e < (1 << (2 * BK)) * 16; e += kThreads) {
    const int code = e >> 4, copy = e & 15;
    const uint32_t c0 = cbs[code & ((1 << BK) - 1)], c1 = cbs[code >> BK];
    uint2 v;
    v.x = (c0 & 0xFFFFu) | (c1 << 16);                // high parts (even, odd coord)
    v.y = (c0 >> 16) | (c1 & 0xFFFF0000u);            // low parts
    *reinterpret_cast<uint2*>(lutK + code * Gm::KSTRIDE + copy * 8) = v;
  }
  if (BV != 2) {
    for (int e = tid; e < (1 << (2 * BV)) * 32; e += kThreads) {
      const int code = e >> 5, copy = e & 31;
      *reinterpret_cast<uint32_t*>(lutV + (code << Gm::VSHIFT) + copy * 4) =
          cbs[16 + (code & ((1 << BV) - 1))] | (cbs[16 + (code >> BV)] << 16);
    }
  }
  // V2 byte tables: low bytes of the 4 fp16 levels, then their high bytes.
  uint32_t vt_lo = 0, vt_hi = 0;
  if (BV == 2) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t h = cbs[16 + j];
      vt_lo |= (h & 0xFFu) << (8 * j);
      vt_hi |= (h >> 8) << (8 * j);
    }
  }

  // Segment search (warp 0) in cost units. The CTAs split a list of
  // (sequence, kv head) segments (sequences in order, kv heads in order
  // within one); a segment of nb > 0 blocks costs nb + sig units, a fixed
  // per-segment overhead sig first, then one unit per block. Finds the first
  // segment holding a block of cost >= at, continuing from the scan state in
  // misc, and writes its descriptor at misc[slot]: b, g, the first block and
  // the number of its blocks with cost in [at, end) (0: none), the segment's
  // block count and length, and the cost of its block 0.
  // len0: this lane's length among the first 32 sequences.
  auto find_segment = [&](long long at, long long end, int len0, int slot) {
    const int sig = misc[kMiscCost + 2];
    int sb = misc[kMiscState];
    long long sP = (long long)(unsigned)misc[kMiscState + 1] | ((long long)misc[kMiscState + 2] << 32);
    while (true) {
      if (sb >= B) {                      // inconsistent lengths: stop this CTA
        if (lane == 0) misc[slot + 3] = 0;
        break;
      }
      const int bb = sb + lane;
      const int len = sb == 0 ? len0 : (bb < B ? min(max(a.ctx_lens[bb], 0), a.cap_tok) : 0);
      const int nb = (len + kBlk - 1) / kBlk;
      const int cst = nb > 0 ? nb + sig : 0;          // cost of one kv head of sequence bb
      int incl = cst;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      const long long segend = (long long)H * (sP + incl);
      const unsigned hit = __ballot_sync(0xFFFFFFFFu, segend > at && bb < B);
      if (hit) {
        const int l = __ffs(hit) - 1;
        const int nbl = __shfl_sync(0xFFFFFFFFu, nb, l);
        const int lenl = __shfl_sync(0xFFFFFFFFu, len, l);
        const int excl = __shfl_sync(0xFFFFFFFFu, incl - cst, l);
        sb += l;
        sP += excl;
        if (lane == 0) {
          const int cl = nbl + sig;
          const long long rel = at - (long long)H * sP;
          const int g = (int)(rel / cl), off = (int)(rel % cl);
          const long long first = (long long)H * sP + (long long)g * cl + sig;
          const int blk0 = max(0, off - sig);
          const long long bend = min((long long)nbl, end - first);
          misc[slot + 0] = sb;
          misc[slot + 1] = g;
          misc[slot + 2] = blk0;
          misc[slot + 3] = (int)max(0LL, bend - blk0);
          misc[slot + 4] = nbl;
          misc[slot + 5] = lenl;
          misc[slot + 6] = (int)(first & 0xFFFFFFFF);
          misc[slot + 7] = (int)(first >> 32);
          misc[kMiscState] = sb;
          misc[kMiscState + 1] = (int)(sP & 0xFFFFFFFF);
          misc[kMiscState + 2] = (int)(sP >> 32);
        }
        break;
      }
      sP += __shfl_sync(0xFFFFFFFFu, incl, 31);
      sb += 32;
    }
  };

  // Balanced split over Geff CTAs, each owning at least one block (the
  // partial count of a sequence relies on it): min(grid, NB), or, when every
  // (sequence, kv head) segment has the same block count and there are no
  // more segments than CTAs, a multiple of the segment count so that no CTA
  // spans two segments.
  auto effective_ctas = [&](long long nbt, int common) {
    int ge = (int)min((long long)Gc, nbt);
    const long long S = (long long)B * H;
    if (common > 0 && S <= Gc) ge = (int)(S * min((long long)(Gc / S), (long long)common));
    return ge;
  };

  // Warp 0: flat block count, whether all sequences have the same length,
  // and the first segment of this CTA (into misc).
  auto plan_cta = [&](int len0) {
    long long tot = 0;
    int nmin = 0x7FFFFFFF, nmax = 0, live = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const bool in = b0 + lane < B;
      const int nb = b0 == 0 ? (len0 + kBlk - 1) / kBlk : (in ? seq_blocks(a, b0 + lane) : 0);
      int sum = nb, lo = in ? nb : 0x7FFFFFFF, hi = nb, nz = nb > 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        lo = min(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
        nz += __shfl_xor_sync(0xFFFFFFFFu, nz, o);
      }
      tot += sum;
      live += nz;
      nmin = min(nmin, lo);
      nmax = max(nmax, hi);
    }
    const long long nbt = tot * H;
    const int common = nmin == nmax ? nmax : -1;
    // no per-segment overhead when every CTA gets a piece of one segment
    const int sig = common > 0 && (long long)B * H <= Gc ? 0 : kSegCost;
    const long long ctot = (tot + (long long)sig * live) * H;
    if (lane == 0) {
      misc[kMiscCost] = (int)(ctot & 0xFFFFFFFF);
      misc[kMiscCost + 1] = (int)(ctot >> 32);
      misc[kMiscCost + 2] = sig;
      misc[kMiscNB] = (int)(nbt & 0xFFFFFFFF);
      misc[kMiscNB + 1] = (int)(nbt >> 32);
      misc[kMiscNB + 2] = common;
      misc[kMiscState] = 0;
      misc[kMiscState + 1] = 0;
      misc[kMiscState + 2] = 0;
      misc[kMiscDesc + 3] = 0;
      misc[kMiscApp] = 0;
    }
    __syncwarp();
    const int ge = effective_ctas(nbt, common);
    if (cta < ge) find_segment(ctot * cta / ge, ctot * (cta + 1) / ge, len0, kMiscDesc);
  };

  // Everything below reads inputs that an earlier launch may have written.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");

  // Lengths of the first 32 sequences, loaded by warp 0 first; the block
  // count and the first segment search use them.
  const int len0 = (warp == 0 && lane < B) ? min(max(a.ctx_lens[lane], 0), a.cap_tok) : 0;
  // The queries (small next to the cache) are pulled into L2 now, spread
  // over the CTAs, so that their later loads do not queue behind the cache
  // stream in DRAM.
  {
    const size_t qbytes = (size_t)B * a.n_q_heads * D * (a.q_dtype == TQ_F32 ? 4 : 2);
    const char* qc = reinterpret_cast<const char*>(a.q);
    for (size_t off = ((size_t)cta * kThreads + tid) * 128; off < qbytes;
         off += (size_t)Gc * kThreads * 128)
      asm volatile("prefetch.global.L2 [%0];\n" ::"l"(qc + off));
    // likewise the decode step's new K/V rows, encoded later by the owner warps
    if (a.new_kv) {
      const size_t kvbytes = (size_t)2 * B * H * D * 2;
      const char* kc = reinterpret_cast<const char*>(a.new_kv);
      for (size_t off = ((size_t)cta * kThreads + tid) * 128; off < kvbytes;
           off += (size_t)Gc * kThreads * 128)
        asm volatile("prefetch.global.L2 [%0];\n" ::"l"(kc + off));
    }
  }

  if (warp == 0) plan_cta(len0);
  __syncthreads();

  const long long NB = (long long)(unsigned)misc[kMiscNB] | ((long long)misc[kMiscNB + 1] << 32);
  const int Geff = effective_ctas(NB, misc[kMiscNB + 2]);
  const long long Ctot = (long long)(unsigned)misc[kMiscCost] | ((long long)misc[kMiscCost + 1] << 32);
  const long long r0 = cta < Geff ? Ctot * cta / Geff : 0;   // this CTA's cost range
  const long long r1 = cta < Geff ? Ctot * (cta + 1) / Geff : 0;
  long long pos = r0;
  unsigned nskip = 0;
  const float log2tau = a.tau > 0.f ? log2f(a.tau) : -INFINITY;

  // ---- status words and empty sequences (CTA 0, one sequence per thread)
  if (cta == 0) {
    for (int b = tid; b < B; b += kThreads) {
      const int raw = a.ctx_lens[b];
      if (a.dev_status && (raw > a.cap_tok || raw <= 0))
        atomicOr(a.dev_status, raw <= 0 ? TQ_DEV_CTX_EMPTY : TQ_DEV_CTX_CLAMPED);
      if (raw <= 0 && a.partial_out) {              // empty slice record
        float* r = reinterpret_cast<float*>(a.out) + (size_t)b * a.n_q_heads * (D + 2);
        for (int h = 0; h < a.n_q_heads; ++h, r += D + 2) {
          for (int i = 0; i < D; i += 2) *reinterpret_cast<float2*>(r + i) = make_float2(0.f, 0.f);
          *reinterpret_cast<float2*>(r + D) = make_float2(-INFINITY, 0.f);
        }
      } else if (raw <= 0) {
        const int es = a.out_dtype == TQ_F32 ? 4 : 2;
        const size_t n16 = (size_t)a.n_q_heads * D * es / 16;
        uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(a.out) +
                                            (size_t)b * a.n_q_heads * D * es);
        for (size_t i = 0; i < n16; ++i) o[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }

  // Lane roles in the score / softmax layout:
  //   NT = 1: the lane holds position gq (tq < 2) or gq + 8 (tq >= 2) of each
  //           16-position step, for heads hs0 = 2·(tq & 1) and hs0 + 1;
  //   NT = 2: positions gq and gq + 8, heads hs0 = 2·tq and hs0 + 1.
  const int hs0 = NT == 1 ? 2 * (tq & 1) : 2 * tq;
  const bool hv0 = hs0 < GQ, hv1 = hs0 + 1 < GQ;
  auto pos_of = [&](int mt, int rr) {
    return 16 * mt + gq + (NT == 1 ? 8 * (tq >> 1) : 8 * rr);
  };

  // Combines the warps' merge buffers into fin[] (GQ x d) and the merged
  // per-head maximum and softmax sum (misc). A buffer holds accumulators in
  // register order (natural = false: lane-major, 32 per lane) or in output
  // order (natural = true), then the per-head maxima and sums.
  float* wts = miscf + kMiscWt;                       // [kWarps][GQ] weights
  auto merge_buffers = [&](bool natural) {
    if (tid < kWarps * GQ) {
      const int w = tid / GQ, h = tid - w * GQ;
      float mx = -INFINITY;
#pragma unroll
      for (int v = 0; v < kWarps; ++v) mx = fmaxf(mx, merge[v * Dd::STRIDE + Dd::M + h]);
      const float mw = merge[w * Dd::STRIDE + Dd::M + h];
      wts[tid] = mw == -INFINITY ? 0.f : fast_exp2(mw - mx);
      if (w == 0) {
        float ls = 0.f;
#pragma unroll
        for (int v = 0; v < kWarps; ++v) {
          const float m = merge[v * Dd::STRIDE + Dd::M + h];
          if (m != -INFINITY) ls += merge[v * Dd::STRIDE + Dd::L + h] * fast_exp2(m - mx);
        }
        miscf[kMiscM + h] = mx;
        miscf[kMiscL + h] = ls;
      }
    }
    __syncthreads();
    for (int i = tid; i < GQ * D; i += kThreads) {
      const int h = i / D;
      const int idx = natural ? i : pv_slot<BV, D>(i - h * D, h);
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) sum += merge[w * Dd::STRIDE + idx] * wts[w * GQ + h];
      fin[i] = sum;
    }
    __syncthreads();
  };

  // Warps split a segment into ranges of whole units: 64-position blocks
  // with the sparse-V gate (its block maximum needs the whole block), else
  // 32 positions, which evens out the shares when a segment has only a few
  // blocks per warp (measured on the decode step too: 795 us per 32-layer
  // step against 814 us with whole blocks). A warp walks its range in
  // chunks of up to 64 positions starting at wp0. The range of warp w in the
  // segment described at misc[slot]:
  const int unit = a.tau > 0.f ? kBlk : kBlk / 2;
  auto warp_share = [&](int slot, int w, int& wp0, int& wp1) {
    const int blk0 = misc[slot + 2], nseg = misc[slot + 3], L = misc[slot + 5];
    const int sp0 = blk0 * kBlk, sp1 = min(L, (blk0 + nseg) * kBlk);
    const int nun = nseg > 0 ? (sp1 - sp0 + unit - 1) / unit : 0;
    wp0 = sp0 + unit * (int)((long long)nun * w / kWarps);
    wp1 = min(sp1, sp0 + unit * (int)((long long)nun * (w + 1) / kWarps));
  };

  int seg_iter = 0;                                   // segments this CTA has done
  while (pos < r1) {
    if (seg_iter > 0) {
      if (warp == 0) find_segment(pos, r1, len0, kMiscDesc);
      __syncthreads();
    }
    const int cs = kMiscDesc;
    const int b = misc[cs + 0], g = misc[cs + 1], blk0 = misc[cs + 2];
    const int nseg = misc[cs + 3], nbl = misc[cs + 4], L = misc[cs + 5];
    if (nseg <= 0) break;
    // cost of the segment's block 0, and the cost just past this CTA's piece
    const long long seg_first = (long long)(unsigned)misc[cs + 6] | ((long long)misc[cs + 7] << 32);
    const long long next_pos = seg_first + blk0 + nseg;

    // query values of the group (warp h < g loads head h), issued before the
    // block loads
    // query head h of the group: coordinates QPL·lane .. QPL·lane + QPL - 1
    auto load_q = [&](int h, float (&qr)[QPL]) {
      const size_t qo = ((size_t)b * a.n_q_heads + (size_t)g * GQ + h) * D + QPL * lane;
      if (a.q_dtype == TQ_F32) {
        const float2* src = reinterpret_cast<const float2*>(reinterpret_cast<const float*>(a.q) + qo);
#pragma unroll
        for (int k = 0; k < QPL / 2; ++k) {
          const float2 v = src[k];
          qr[2 * k] = v.x;
          qr[2 * k + 1] = v.y;
        }
      } else {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint16_t*>(a.q) + qo);
        const bool bf = a.q_dtype == TQ_BF16;
#pragma unroll
        for (int k = 0; k < QPL / 2; ++k) {
          const float2 f = unpack16x2(src[k], bf);
          qr[2 * k] = f.x;
          qr[2 * k + 1] = f.y;
        }
      }
    };
    float qraw[QPL];
#pragma unroll
    for (int k = 0; k < QPL; ++k) qraw[k] = 0.f;
    if (warp < GQ) load_q(warp, qraw);

    // ---- this warp's share of the segment
    const int sp0 = blk0 * kBlk, sp1 = min(L, (blk0 + nseg) * kBlk);
    const int nun = (sp1 - sp0 + unit - 1) / unit;
    int wp0, wp1;
    warp_share(cs, warp, wp0, wp1);
    const int nw = wp1 > wp0 ? (wp1 - wp0 + kBlk - 1) / kBlk : 0;

    float acc[NPV][4];
#pragma unroll
    for (int r = 0; r < NPV; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    unsigned nsk0 = 0, nsk1 = 0;               // gated positions of heads hs0, hs0 + 1

    const size_t seq_row = ((size_t)b * H + g) * a.cap_tok;
    const uint8_t* gk = a.packed_k + seq_row * Gm::RK;
    const uint8_t* gv = a.packed_v + seq_row * Gm::RV;
    const uint16_t* gnk = a.norms_k + seq_row;
    const uint16_t* gnv = a.norms_v + seq_row;
    const uint32_t wring = Gm::FIXED + warp * Gm::NSTAGE * Gm::STAGE;   // smem offset

    // Bulk copies of chunk c of the warp's range (its j-th staged chunk)
    // into ring slot j % NSTAGE, issued by lane 0: K rows, V rows and the
    // two norm runs are contiguous in global memory. Rows past the range are
    // not copied; their slot bytes are stale and masked out below (norms are
    // copied in whole 16-byte runs, which stay inside cap_tok).
    // ... of chunk c of warp v's range [v0, v1) into slot j % NSTAGE of v's
    // ring (v = this warp, or in the first segment a query-rotating warp
    // whose first copies another warp issues)
    auto issue_for = [&](int v, int v0, int v1, int c, int j) {
      if (lane == 0) {
        const int t0 = v0 + c * kBlk;
        const int rows = min(kBlk, v1 - t0);
        // A bulk copy moves a multiple of 16 bytes: row counts are rounded up
        // to Gm::KROWS / VROWS (2 for the 24-byte rows at d = 64 and 3 bits,
        // else 1) and norm runs to 8; every bound stays inside cap_tok, a
        // multiple of 8.
        const int krows = min(kBlk, (rows + Gm::KROWS - 1) / Gm::KROWS * Gm::KROWS);
        const int vrows = min(kBlk, (rows + Gm::VROWS - 1) / Gm::VROWS * Gm::VROWS);
        const int nrows = min(kBlk, (rows + 7) & ~7);
        const int slot = j % Gm::NSTAGE;
        const uint32_t dst = smem_addr(smem) + Gm::FIXED + (v * Gm::NSTAGE + slot) * Gm::STAGE;
        const uint32_t bar = smem_addr(smem) + Gm::QOFF + Gm::QS + Gm::MISC + (v * kMaxStages + slot) * 8;
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        const uint32_t extra = kInjectWaitFaults && a.new_kv == nullptr && j == 0 ? 16u : 0u;
        // the rows lie in the sequence's capacity (checked in the
        // bounds-checked build; a skipped copy still completes the phase)
        const bool inb = tq_check(t0 >= 0 && rows > 0 &&
                                  t0 + max(krows, max(vrows, nrows)) <= a.cap_tok, a.dev_status);
        mbar_expect(bar, inb ? krows * Gm::RK + vrows * Gm::RV + 4 * nrows + extra : 0u);
        if (inb) {
          bulk_g2s(dst, gk + (size_t)t0 * Gm::RK, krows * Gm::RK, bar);
          bulk_g2s(dst + Gm::KB, gv + (size_t)t0 * Gm::RV, vrows * Gm::RV, bar);
          bulk_g2s(dst + Gm::NKOFF, gnk + t0, 2 * nrows, bar);
          bulk_g2s(dst + Gm::NKOFF + 2 * kBlk, gnv + t0, 2 * nrows, bar);
        }
      }
    };
    auto issue = [&](int c, int j) { issue_for(warp, wp0, wp1, c, j); };

    // every slot of the ring gets a block (or an empty group); the warps
    // that rotate the query fill theirs afterwards, so that the query loads
    // do not wait behind their block loads
    auto fill_ring = [&]() {
#pragma unroll
      for (int p = 0; p < Gm::NSTAGE; ++p)
        if (!stalled && p < nw) issue(p, jdone + p);
    };
    int issued = stalled ? 0 : min(nw, Gm::NSTAGE);
    auto bar_of = [&](int jj) { return wbar + 8 * (jj % Gm::NSTAGE); };
    auto par_of = [&](int jj) { return (uint32_t)(jj / Gm::NSTAGE) & 1u; };
    // In the first segment every ring starts at chunk 0, so the warps that
    // do not rotate the query also issue the first chunks of those that do
    // (query warp v by warp GQ + v % (warps - GQ)): all rings fill at once.
    const bool proxy_fill = seg_iter == 0 && GQ < kWarps;
    if (warp >= GQ) {
      fill_ring();
      if (proxy_fill)
        for (int v = warp - GQ; v < GQ; v += kWarps - GQ) {
          int v0, v1;
          warp_share(cs, v, v0, v1);
          const int nv_ = v1 > v0 ? (v1 - v0 + kBlk - 1) / kBlk : 0;
          for (int p = 0; p < Gm::NSTAGE && p < nv_; ++p) issue_for(v, v0, v1, p, p);
        }
    }
    // ---- rotated query of the group: warp w handles query heads w, w +
    // kWarps, ... (the first one's values are already loaded)
    auto rotate_q = [&](int h, const float (&qr)[QPL]) {
      float x[QPL];
#pragma unroll
      for (int k = 0; k < QPL; ++k) {
        const int c = QPL * lane + k;
        x[k] = apply_sign(qr[k], sm.w[c >> 5], c & 31);
      }
      fwht_warp<QPL>(x, lane);
      // log2(e)/d^{3/2} folds the rotation normalization, the codebook's
      // 1/sqrt(d) and the softmax 1/sqrt(d); a power-of-two scale keeps the
      // fp16 high part near 2^14 so that the low part stays normal.
      float amax = 0.f;
#pragma unroll
      for (int k = 0; k < QPL; ++k) {
        x[k] *= kLog2e / ((float)D * Dd::ROOT);
        amax = fmaxf(amax, fabsf(x[k]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      const int e = amax > 0.f ? ilogbf(amax) : 0;
      const float qs = ldexpf(1.f, min(14 - e, 120));
      uint32_t* hdst = reinterpret_cast<uint32_t*>(qhi + h * D + QPL * lane);
      uint32_t* ldst = reinterpret_cast<uint32_t*>(qlo + h * D + QPL * lane);
#pragma unroll
      for (int k = 0; k < QPL; k += 2) {
        const float v0 = x[k] * qs, v1 = x[k + 1] * qs;
        const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
        hdst[k / 2] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
        ldst[k / 2] = pack_half2(v0 - __half2float(h0), v1 - __half2float(h1));
      }
      if (lane == 0) miscf[kMiscQInv + h] = 1.f / (qs * kKScale);
    };
    if (warp < GQ) {
      rotate_q(warp, qraw);
      for (int h = warp + kWarps; h < GQ; h += kWarps) {
        float q2[QPL];
        load_q(h, q2);
        rotate_q(h, q2);
      }
      if (!proxy_fill) fill_ring();
    }
    // ---- decode-step append. The owner warp (its range ends at the
    // sequence's last position) patches the new row into its staged last
    // chunk. The encode of the new token of (b, g) (lanes 0-3: K, 4-7: V;
    // the encode kernel's per-vector code), the store of cache row L - 1 and
    // the copy for the patch are done by a helper warp with the fewest
    // blocks, which hands the row over through shared memory.
    const bool app_cta = a.new_kv != nullptr && blk0 + nseg == nbl && sp1 == L && nun > 0;
    const bool app = app_cta && nw > 0 && wp1 == L;
    int helper = -1;
    if (app_cta) {
      int owner_w = 0, best = 1 << 30;
#pragma unroll 1
      for (int w = 0; w < kWarps; ++w)
        if ((long long)nun * (w + 1) / kWarps > (long long)nun * w / kWarps) owner_w = w;
#pragma unroll 1
      for (int w = 0; w < kWarps; ++w) {
        const int cw = (int)((long long)nun * (w + 1) / kWarps - (long long)nun * w / kWarps);
        if (w != owner_w && cw < best) {
          best = cw;
          helper = w;
        }
      }
      if (helper < 0) helper = owner_w;
    }
    uint8_t* app_k = smem + Gm::APPOFF;
    uint8_t* app_v = app_k + D / 2;
    uint16_t* app_n = reinterpret_cast<uint16_t*>(app_k + D);
    __syncthreads();
    // The helper encodes after the CTA barrier: only the owner needs the new
    // row, for its last chunk, and the helper has the fewest blocks.
    if (app_cta && warp == helper) {
      constexpr int LPV = D / 32;                     // lanes per vector
      if (lane < 2 * LPV) {
        const int sub = lane & (LPV - 1);
        const bool isv = lane >= LPV;
        uint32_t smask[16];
        sign_masks(sm, sub, smask);
        const uint16_t* src = a.new_kv + ((size_t)((isv ? B : 0) + b) * H + g) * D;
        float x[32];
        load_signed(src, sub, a.new_kv_bf16 != 0, smask, x);
        const unsigned gmask = ((1u << LPV) - 1u) << (lane & ~(LPV - 1));
        if (isv)
          encode_vector<BV, LPV>(x, cbv, sub, gmask, app_v, app_n + 1, a.dev_status);
        else
          encode_vector<BK, LPV>(x, cbk, sub, gmask, app_k, app_n, a.dev_status);
      }
      __syncwarp();
      const size_t row = seq_row + (size_t)(L - 1);
      for (int i = lane; i < Gm::RK / 4; i += 32)
        reinterpret_cast<uint32_t*>(a.packed_k + row * Gm::RK)[i] =
            reinterpret_cast<const uint32_t*>(app_k)[i];
      for (int i = lane; i < Gm::RV / 4; i += 32)
        reinterpret_cast<uint32_t*>(a.packed_v + row * Gm::RV)[i] =
            reinterpret_cast<const uint32_t*>(app_v)[i];
      if (lane == 0) {
        a.norms_k[row] = app_n[0];
        a.norms_v[row] = app_n[1];
        __threadfence_block();                        // the row before the flag
        if (!kInjectWaitFaults) *reinterpret_cast<volatile int*>(misc + kMiscApp) = seg_iter + 1;
      }
    }

    // ---- query fragments (B operand of the score MMA), column n = gq.
    //   NT = 1: columns 0-3 hold the high part of heads 0-3, 4-7 their low part.
    //   NT = 2: tile 0 column n = high part of head n, tile 1 = low part.
    uint32_t qb[NT][KS][2];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int head = NT == 1 ? (gq & 3) : gq;
      const __half* src = (NT == 1 ? (gq < 4) : (t == 0)) ? qhi : qlo;
      const bool ok = head < GQ;
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        const int c0 = (D / 4) * tq + 4 * s;
        qb[t][s][0] = ok ? *reinterpret_cast<const uint32_t*>(src + head * D + c0) : 0u;
        qb[t][s][1] = ok ? *reinterpret_cast<const uint32_t*>(src + head * D + c0 + 2) : 0u;
      }
    }
    // Query scale of heads hs0, hs0 + 1. A head beyond the group has a zero
    // query and scale 1: its scores are 0 and its weights finite, and its
    // accumulator columns are never read.
    const float2 sinv = make_float2(hv0 ? miscf[kMiscQInv + hs0] : 1.f,
                                    hv1 ? miscf[kMiscQInv + hs0 + 1] : 1.f);
    const bool gate = a.tau > 0.f;

    for (int i = 0; i < nw && !stalled; ++i) {
      const int j = jdone + i;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar_of(j), par_of(j)))) {
        // give up: report, wait (bounded) for the copies still in flight,
        // issue nothing more
        stalled = true;
        if (lane == 0 && a.dev_status) atomicOr(a.dev_status, TQ_DEV_WAIT_TIMEOUT);
        for (int k = i + 1; k < issued; ++k) mbar_wait(bar_of(jdone + k), par_of(jdone + k));
        __syncwarp();
        break;
      }
      const uint32_t st = wring + (j % Gm::NSTAGE) * Gm::STAGE;         // smem offset
      const int t0 = wp0 + i * kBlk;                // chunk [t0, cend)
      const int cend = min(wp1, t0 + kBlk);
      const bool partial = cend < t0 + kBlk;
      if (app && cend == L) {                       // the staged row L - 1 is stale
        if (lane == 0) {                              // wait (bounded) for the helper
          if (*reinterpret_cast<volatile int*>(misc + kMiscApp) != seg_iter + 1 &&
              !wait_flag_slow(misc + kMiscApp, seg_iter + 1) && a.dev_status)
            atomicOr(a.dev_status, TQ_DEV_WAIT_TIMEOUT);
          __threadfence_block();
        }
        __syncwarp();
        const int r = L - 1 - t0;
        for (int w = lane; w < Gm::RK / 4; w += 32)
          *reinterpret_cast<uint32_t*>(smem + st + r * Gm::RK + 4 * w) =
              reinterpret_cast<const uint32_t*>(app_k)[w];
        for (int w = lane; w < Gm::RV / 4; w += 32)
          *reinterpret_cast<uint32_t*>(smem + st + Gm::KB + r * Gm::RV + 4 * w) =
              reinterpret_cast<const uint32_t*>(app_v)[w];
        if (lane == 0) {
          *reinterpret_cast<uint16_t*>(smem + st + Gm::NKOFF + 2 * r) = app_n[0];
          *reinterpret_cast<uint16_t*>(smem + st + Gm::NKOFF + 2 * kBlk + 2 * r) = app_n[1];
        }
        __syncwarp();
      }

      // -- scores: 4 steps of 16 positions, each as two 8-position groups.
      // A operand rows 0-7 are the K codebook high parts of the group's
      // positions, rows 8-15 the low parts of the same positions, so one
      // table entry (high pair, low pair) fills two adjacent fragment
      // registers; D rows r and r + 8 add up to the score of position r.
      float sc[4][NR][2];               // [step][row][head hs0 + e]
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        if (16 * mt >= cend - t0) {          // step past the chunk: all masked
#pragma unroll
          for (int rr = 0; rr < NR; ++rr) sc[mt][rr][0] = sc[mt][rr][1] = -INFINITY;
          continue;
        }
        uint32_t kw[2][(CBK + 3) / 4 + 1];   // positions gq and gq + 8, chunk tq
#pragma unroll
        for (int gr = 0; gr < 2; ++gr)
          load_chunk<CBK>(smem, st + (16 * mt + 8 * gr + gq) * Gm::RK + CBK * tq, kw[gr]);
        float d[2][NT][4];
#pragma unroll
        for (int gr = 0; gr < 2; ++gr)
#pragma unroll
          for (int t = 0; t < NT; ++t) d[gr][t][0] = d[gr][t][1] = d[gr][t][2] = d[gr][t][3] = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2) {
#pragma unroll
          for (int gr = 0; gr < 2; ++gr) {
            uint32_t a0, a1;
            if constexpr (Gm::KWIDE) {               // (code << 8) | lane offset
              a0 = __byte_perm(kw[gr][s2 >> 1], lbK, 0x7604u | (uint32_t)((2 * s2) & 3) << 4);
              a1 = __byte_perm(kw[gr][s2 >> 1], lbK, 0x7604u | (uint32_t)((2 * s2 + 1) & 3) << 4);
            } else {
              a0 = k_entry<BK>(kw[gr], 2 * s2) + lbK;
              a1 = k_entry<BK>(kw[gr], 2 * s2 + 1) + lbK;
            }
            const uint2 e0 = lds<uint2>(smem, a0);
            const uint2 e1 = lds<uint2>(smem, a1);
#pragma unroll
            for (int t = 0; t < NT; ++t)
              mma16816(d[gr][t], e0.x, e0.y, e1.x, e1.y, qb[t][s2][0], qb[t][s2][1]);
          }
        }
        if (NT == 1) {
          // Columns 2tq, 2tq+1: the high part of heads 2tq, 2tq+1 (tq < 2) or
          // the low part of heads 2(tq-2), +1 (tq >= 2); lane ^ 2 holds the
          // other part. Lanes tq < 2 keep group 0, tq >= 2 keep group 1.
          const float a0 = d[0][0][0] + d[0][0][2], a1 = d[0][0][1] + d[0][0][3];
          const float c0 = d[1][0][0] + d[1][0][2], c1 = d[1][0][1] + d[1][0][3];
          const bool lowq = tq >= 2;
          const float s0 = __shfl_xor_sync(0xFFFFFFFFu, lowq ? a0 : c0, 2);
          const float s1 = __shfl_xor_sync(0xFFFFFFFFu, lowq ? a1 : c1, 2);
          sc[mt][0][0] = (lowq ? c0 : a0) + s0;
          sc[mt][0][1] = (lowq ? c1 : a1) + s1;
        } else {
#pragma unroll
          for (int gr = 0; gr < 2; ++gr) {
            sc[mt][gr][0] = (d[gr][0][0] + d[gr][0][2]) + d[gr][NT - 1][0];
            sc[mt][gr][1] = (d[gr][0][1] + d[gr][0][3]) + d[gr][NT - 1][1];
          }
        }
      }
      // -- scores x = (MMA sum) · n_K per position and head (the query scale
      // is applied below), masked past the chunk; block maximum per head
      auto scale_scores = [&](auto part_c) {          // sc <- x, in place
        constexpr bool PART = decltype(part_c)::value;
        float2 xm = make_float2(-INFINITY, -INFINITY);
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
          for (int rr = 0; rr < NR; ++rr) {
            const int p = pos_of(mt, rr);
            const float nk = __half2float(__ushort_as_half(lds<uint16_t>(smem, st + Gm::NKOFF + 2 * p)));
            float2 x = __fmul2_rn(make_float2(sc[mt][rr][0], sc[mt][rr][1]), make_float2(nk, nk));
            if (PART && t0 + p >= cend) x = make_float2(-INFINITY, -INFINITY);
            sc[mt][rr][0] = x.x;
            sc[mt][rr][1] = x.y;
            xm.x = fmaxf(xm.x, x.x);
            xm.y = fmaxf(xm.y, x.y);
          }
        return xm;
      };
      float2 xm = partial ? scale_scores(std::true_type{}) : scale_scores(std::false_type{});
      // lanes holding the same heads: NT = 1 -> lane bits 1-4; NT = 2 -> bits 2-4
#pragma unroll
      for (int o = (NT == 1 ? 2 : 4); o < 32; o <<= 1) {
        xm.x = fmaxf(xm.x, __shfl_xor_sync(0xFFFFFFFFu, xm.x, o));
        xm.y = fmaxf(xm.y, __shfl_xor_sync(0xFFFFFFFFu, xm.y, o));
      }
      // block maximum of the scores s = x · scale (the scale is positive, so
      // the maximum of the rounded products is the rounded product of the maximum)
      const float2 mb = __fmul2_rn(xm, sinv);
      const float mn0 = fmaxf(m_run[0], mb.x), mn1 = fmaxf(m_run[1], mb.y);
      const float al0 = fast_exp2(m_run[0] - mn0), al1 = fast_exp2(m_run[1] - mn1);
      m_run[0] = mn0;
      m_run[1] = mn1;
      l_run[0] *= al0;
      l_run[1] *= al1;

      // -- weights w = 2^(s - m), P' = w · n_V packed as fp16 pairs (heads hs0,
      // hs0+1). With the sparse-V gate, P' = 0 where 2^(s - M_blk) < tau.
      uint32_t pk[4][NR];
      auto weights = [&](auto gate_c, auto part_c) {
        constexpr bool GATE = decltype(gate_c)::value, PART = decltype(part_c)::value;
        const float2 negm = make_float2(-mn0, -mn1);
        float2 lsum = make_float2(0.f, 0.f);
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
          for (int rr = 0; rr < NR; ++rr) {
            const int p = pos_of(mt, rr);
            const float nv = __half2float(__ushort_as_half(lds<uint16_t>(smem, st + Gm::NKOFF + 2 * kBlk + 2 * p)));
            float2 e, sv;
            if (GATE) {                             // the rounded score, as the gate compares it
              sv = __fmul2_rn(make_float2(sc[mt][rr][0], sc[mt][rr][1]), sinv);
              e = __fadd2_rn(sv, negm);
            } else {
              e = __ffma2_rn(make_float2(sc[mt][rr][0], sc[mt][rr][1]), sinv, negm);
            }
            const float2 w = make_float2(fast_exp2(e.x), fast_exp2(e.y));
            lsum = __fadd2_rn(lsum, w);
            float2 pp = __fmul2_rn(w, make_float2(nv, nv));
            if (GATE) {
              const bool g0 = sv.x - mb.x < log2tau, g1 = sv.y - mb.y < log2tau;   // exp(s - M_blk) < tau
              if (g0) pp.x = 0.f;
              if (g1) pp.y = 0.f;
              nsk0 += g0 && hv0 && sv.x != -INFINITY;
              nsk1 += g1 && hv1 && sv.y != -INFINITY;
            }
            if (PART && t0 + p >= cend) pp = make_float2(0.f, 0.f);   // stale slot bytes
            pk[mt][rr] = pack_half2(pp.x, pp.y);
          }
        l_run[0] += lsum.x;
        l_run[1] += lsum.y;
      };
      if (gate) {
        if (partial) weights(std::true_type{}, std::true_type{});
        else weights(std::true_type{}, std::false_type{});
      } else {
        if (partial) weights(std::false_type{}, std::true_type{});
        else weights(std::false_type{}, std::false_type{});
      }
      // rescale the PV accumulators (PV layout: heads 2tq, 2tq+1)
      {
        float2 al = make_float2(al0, al1);
        if (NT == 1 && tq >= 2) al = make_float2(1.f, 1.f);   // heads 4-7: padding
        if (__any_sync(0xFFFFFFFFu, al.x != 1.f || al.y != 1.f)) {
#pragma unroll
          for (int r = 0; r < NPV; ++r) {
            const float2 u = __fmul2_rn(make_float2(acc[r][0], acc[r][1]), al);
            const float2 v = __fmul2_rn(make_float2(acc[r][2], acc[r][3]), al);
            acc[r][0] = u.x;
            acc[r][1] = u.y;
            acc[r][2] = v.x;
            acc[r][3] = v.y;
          }
        }
      }

      // -- P·V over the four 16-position steps
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        if (16 * mt >= cend - t0) break;     // steps past the chunk
        uint32_t x0, x1;   // P' of positions 0-7 / 8-15 x heads 0-7, standard layout
        if (NT == 1) {
          const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, pk[mt][0], 2);
          x0 = tq < 2 ? pk[mt][0] : 0u;
          x1 = tq < 2 ? other : 0u;
        } else {
          x0 = pk[mt][0];
          x1 = pk[mt][NR - 1];
        }
        if (gate && !__any_sync(0xFFFFFFFFu, (x0 | x1) != 0u)) continue;   // whole step gated
        const uint32_t b0 = transpose8x8(x0), b1 = transpose8x8(x1);
        if (BV == 2) {
          // lane gq reads D/32 bytes (D/8 coordinates) of the rows of
          // positions 2tq, 2tq+1, 2tq+8, 2tq+9; xab/xcd interleave them by
          // byte, NH = D/64 words each
          constexpr int NB = D / 32, NH = D / 64;
          const uint32_t vrow = st + Gm::KB + (16 * mt + 2 * tq) * Gm::RVS + NB * gq;
          uint32_t wA[(NB + 3) / 4], wB[(NB + 3) / 4], wC[(NB + 3) / 4], wD[(NB + 3) / 4];
#pragma unroll
          for (int q4 = 0; q4 < (NB + 3) / 4; ++q4) {
            if constexpr (NB == 2) {
              wA[q4] = lds<uint16_t>(smem, vrow);
              wB[q4] = lds<uint16_t>(smem, vrow + Gm::RVS);
              wC[q4] = lds<uint16_t>(smem, vrow + 8 * Gm::RVS);
              wD[q4] = lds<uint16_t>(smem, vrow + 9 * Gm::RVS);
            } else {
              wA[q4] = lds<uint32_t>(smem, vrow + 4 * q4);
              wB[q4] = lds<uint32_t>(smem, vrow + Gm::RVS + 4 * q4);
              wC[q4] = lds<uint32_t>(smem, vrow + 8 * Gm::RVS + 4 * q4);
              wD[q4] = lds<uint32_t>(smem, vrow + 9 * Gm::RVS + 4 * q4);
            }
          }
          uint32_t xab[NH], xcd[NH];
#pragma unroll
          for (int hh = 0; hh < NH; ++hh) {
            const uint32_t sel = (hh & 1) ? 0x7362u : 0x5140u;
            xab[hh] = __byte_perm(wA[hh >> 1], wB[hh >> 1], sel);
            xcd[hh] = __byte_perm(wC[hh >> 1], wD[hh >> 1], sel);
          }
#pragma unroll
          for (int half = 0; half < NH; ++half) {
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
          uint32_t v0[(CBV + 3) / 4 + 1], v1[(CBV + 3) / 4 + 1];
          const uint32_t r0p = st + Gm::KB + (16 * mt + gq) * Gm::RVS + CBV * tq;
          load_chunk<CBV>(smem, r0p, v0);
          load_chunk<CBV>(smem, r0p + 8 * Gm::RVS, v1);
#pragma unroll
          for (int r = 0; r < NPV; ++r) {
            const uint32_t y0 = lds<uint32_t>(smem, pair_code_shifted<BV, Gm::VSHIFT>(v0, 2 * r) | lbV);
            const uint32_t y1 = lds<uint32_t>(smem, pair_code_shifted<BV, Gm::VSHIFT>(v0, 2 * r + 1) | lbV);
            const uint32_t y2 = lds<uint32_t>(smem, pair_code_shifted<BV, Gm::VSHIFT>(v1, 2 * r) | lbV);
            const uint32_t y3 = lds<uint32_t>(smem, pair_code_shifted<BV, Gm::VSHIFT>(v1, 2 * r + 1) | lbV);
            mma16816(acc[r], transpose8x8(y0), transpose8x8(y1), transpose8x8(y2),
                     transpose8x8(y3), b0, b1);
          }
        }
      }
      __syncwarp();                                  // the slot is free again
      if (i + Gm::NSTAGE < nw) {
        issue(i + Gm::NSTAGE, j + Gm::NSTAGE);
        ++issued;
      }
    }
    jdone += nw;
    nskip += nsk0 + nsk1;
    if (a.head_skipped && gate) {             // per (sequence, query head) gate counts
#pragma unroll
      for (int o = (NT == 1 ? 2 : 4); o < 32; o <<= 1) {
        nsk0 += __shfl_xor_sync(0xFFFFFFFFu, nsk0, o);
        nsk1 += __shfl_xor_sync(0xFFFFFFFFu, nsk1, o);
      }
      if (gq == 0 && (NT == 2 || tq < 2)) {
        unsigned int* hk = a.head_skipped + (size_t)b * a.n_q_heads + (size_t)g * GQ + hs0;
        if (hv0 && nsk0) atomicAdd(hk, nsk0);
        if (hv1 && nsk1) atomicAdd(hk + 1, nsk1);
      }
    }

    // ---- per-warp softmax sums over the lanes holding the same heads
#pragma unroll
    for (int o = (NT == 1 ? 2 : 4); o < 32; o <<= 1) {
      l_run[0] += __shfl_xor_sync(0xFFFFFFFFu, l_run[0], o);
      l_run[1] += __shfl_xor_sync(0xFFFFFFFFu, l_run[1], o);
    }

    // ---- merge the warps of this segment. Each warp leaves its partial in
    // a merge buffer (accumulators as stored in its registers, then the
    // per-head maximum and sum); the buffers are combined per output element.
    __syncthreads();                                  // all warps done with the ring
    {
      float* wm = merge + warp * Dd::STRIDE;
      if (gq == 0 && (NT == 2 || tq < 2)) {
        if (hv0) {
          wm[Dd::M + hs0] = nw > 0 ? m_run[0] : -INFINITY;
          wm[Dd::L + hs0] = nw > 0 ? l_run[0] : 0.f;
        }
        if (hv1) {
          wm[Dd::M + hs0 + 1] = nw > 0 ? m_run[1] : -INFINITY;
          wm[Dd::L + hs0 + 1] = nw > 0 ? l_run[1] : 0.f;
        }
      }
#pragma unroll
      for (int r = 0; r < NPV; ++r)
        *reinterpret_cast<float4*>(wm + lane * Dd::LANE + 4 * r) =
            make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
    }
    __syncthreads();
    merge_buffers(false);

    bool finalize = nseg == nbl;                      // this CTA saw the whole sequence
    if (!finalize) {
      const int sigma = b * H + g;
      const long long last = seg_first + nbl - 1;
      const int c_first = cta_of(seg_first, Ctot, Geff), c_last = cta_of(last, Ctot, Geff);
      const int n_parts = c_last - c_first + 1;
      float* slot = a.slots + (size_t)(cta + sigma) * GQ * (D + 2);
      for (int i = tid; i < GQ * D; i += kThreads) slot[i] = fin[i];
      if (tid < GQ) {
        slot[GQ * D + 2 * tid] = miscf[kMiscM + tid];
        slot[GQ * D + 2 * tid + 1] = miscf[kMiscL + tid];
      }
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        const int prev = atomicAdd(a.counters + sigma, 1);
        const bool is_last = prev == n_parts - 1;
        if (is_last) __threadfence();
        misc[kMiscLast] = is_last;
      }
      __syncthreads();
      finalize = misc[kMiscLast] != 0;
      if (finalize) {
        // Merge the n_parts partials of this sequence: warp w folds partials
        // w, w + kWarps, ... (two per round of loads) into a merge buffer in
        // output order, kFinChunk outputs per lane per pass, then the buffers
        // are combined as above.
        const float* s0 = a.slots + (size_t)(c_first + sigma) * GQ * (D + 2);
        const size_t stride = (size_t)GQ * (D + 2);
        const int nk = GQ * D / 32;                   // outputs per lane: lane + 32k
        float* wm = merge + warp * Dd::STRIDE;
        constexpr int kFinChunk = 16;
        for (int k0 = 0; k0 < nk; k0 += kFinChunk) {
          float S[kFinChunk];
          float Mh = -INFINITY, Lh = 0.f;             // lane h < GQ: head h
#pragma unroll
          for (int k = 0; k < kFinChunk; ++k) S[k] = 0.f;
          for (int p = warp; p < n_parts; p += 2 * kWarps) {
            const bool two = p + kWarps < n_parts;
            const float* pa = s0 + (size_t)p * stride;
            const float* pb = s0 + (size_t)(two ? p + kWarps : p) * stride;
            float va[kFinChunk], vb[kFinChunk];
#pragma unroll
            for (int k = 0; k < kFinChunk; ++k) {
              const bool ok = k0 + k < nk;
              va[k] = ok ? __ldcg(pa + lane + 32 * (k0 + k)) : 0.f;
              vb[k] = ok && two ? __ldcg(pb + lane + 32 * (k0 + k)) : 0.f;
            }
            const bool hl = lane < GQ;
            const float ma = hl ? __ldcg(pa + GQ * D + 2 * lane) : -INFINITY;
            const float la = hl ? __ldcg(pa + GQ * D + 2 * lane + 1) : 0.f;
            const float mb = hl && two ? __ldcg(pb + GQ * D + 2 * lane) : -INFINITY;
            const float lb = hl && two ? __ldcg(pb + GQ * D + 2 * lane + 1) : 0.f;
            // per head (lane h): new maximum and the three rescale factors
            const float Mn = fmaxf(Mh, fmaxf(ma, mb));
            const float fo = Mh == -INFINITY ? 0.f : fast_exp2(Mh - Mn);
            const float fa = ma == -INFINITY ? 0.f : fast_exp2(ma - Mn);
            const float fb = mb == -INFINITY ? 0.f : fast_exp2(mb - Mn);
            Lh = Lh * fo + la * fa + lb * fb;
            Mh = Mn;
#pragma unroll
            for (int k = 0; k < kFinChunk; ++k) {
              const int h = min((k0 + k) / (D / 32), kMaxGroup - 1);   // head of lane + 32k
              const float go = __shfl_sync(0xFFFFFFFFu, fo, h);
              const float ga = __shfl_sync(0xFFFFFFFFu, fa, h);
              const float gb = __shfl_sync(0xFFFFFFFFu, fb, h);
              S[k] = S[k] * go + va[k] * ga + vb[k] * gb;
            }
          }
#pragma unroll
          for (int k = 0; k < kFinChunk; ++k)
            if (k0 + k < nk) wm[lane + 32 * (k0 + k)] = S[k];
          if (k0 == 0 && lane < GQ) {
            wm[Dd::M + lane] = Mh;
            wm[Dd::L + lane] = Lh;
          }
        }
        __syncthreads();
        merge_buffers(true);
        if (tid == 0) atomicExch(a.counters + sigma, 0);
      }
    }
    for (int h = warp; finalize && a.partial_out && h < GQ; h += kWarps) {
      // context-parallel slice: the record (acc, base-2 maximum, sum)
      float* r = reinterpret_cast<float*>(a.out) +
                 ((size_t)b * a.n_q_heads + (size_t)g * GQ + h) * (D + 2);
#pragma unroll
      for (int k = 0; k < QPL; k += 2)
        *reinterpret_cast<float2*>(r + QPL * lane + k) =
            make_float2(fin[h * D + QPL * lane + k], fin[h * D + QPL * lane + k + 1]);
      if (lane == 0)
        *reinterpret_cast<float2*>(r + D) = make_float2(miscf[kMiscM + h], miscf[kMiscL + h]);
    }
    for (int h = warp; finalize && !a.partial_out && h < GQ; h += kWarps) {
      const float inv_l = 1.f / miscf[kMiscL + h];
      float x[QPL];
#pragma unroll
      for (int k = 0; k < QPL; ++k) x[k] = fin[h * D + QPL * lane + k] * inv_l;
      fwht_warp<QPL>(x, lane);
      const size_t ob = ((size_t)b * a.n_q_heads + (size_t)g * GQ + h) * D + QPL * lane;
#pragma unroll
      for (int k = 0; k < QPL; ++k) {
        const int c = QPL * lane + k;
        x[k] = apply_sign(x[k], sm.w[c >> 5], c & 31) * (1.f / D);
      }
      if (a.out_dtype == TQ_F32) {
        float2* o = reinterpret_cast<float2*>(reinterpret_cast<float*>(a.out) + ob);
#pragma unroll
        for (int k = 0; k < QPL / 2; ++k) o[k] = make_float2(x[2 * k], x[2 * k + 1]);
      } else {
        uint32_t* o = reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(a.out) + ob);
        const bool bf = a.out_dtype == TQ_BF16;
#pragma unroll
        for (int k = 0; k < QPL / 2; ++k) {
          const uint32_t h0 = bf ? f32_to_bf16_bits(x[2 * k]) : f32_to_f16_bits(x[2 * k]);
          const uint32_t h1 = bf ? f32_to_bf16_bits(x[2 * k + 1]) : f32_to_f16_bits(x[2 * k + 1]);
          o[k] = h0 | (h1 << 16);
        }
      }
    }
    pos = next_pos;
    ++seg_iter;
    __syncthreads();                                  // misc / fin / q~ reuse
  }

  if (a.skipped) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nskip += __shfl_xor_sync(0xFFFFFFFFu, nskip, o);
    if (lane == 0 && nskip) atomicAdd(a.skipped, (unsigned long long)nskip);
  }
}

inline int sm_count() {
  static std::atomic<int> cached[64] = {};
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

template <int BK, int BV, int NT, int D>
cudaError_t launch_one(const AttendArgs& a, const Codebook& cbk, const Codebook& cbv,
                       const SignMask& sm, int n_ctas, cudaStream_t stream) {
  using Gm = Geo<BK, BV, D>;
  // set once per device (idempotent; atomic so that concurrent first calls do not race)
  static std::atomic<bool> configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(attend_kernel<BK, BV, NT, D>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, Gm::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  const int grid = n_ctas > 0 ? n_ctas : Gm::PER_SM * sm_count();
  // Programmatic dependent launch: the kernel's set-up may overlap the tail
  // of the previous launch in the stream; it waits for that launch before
  // reading any input (griddepcontrol.wait).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(32 * Gm::NW);
  cfg.dynamicSmemBytes = Gm::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attend_kernel<BK, BV, NT, D>, a, cbk, cbv, sm);
}

template <int BK, int BV, int D>
cudaError_t launch_pair(const AttendArgs& a, const Codebook& cbk, const Codebook& cbv,
                        const SignMask& sm, int n_ctas, cudaStream_t stream) {
  return a.gqa <= 4 ? launch_one<BK, BV, 1, D>(a, cbk, cbv, sm, n_ctas, stream)
                    : launch_one<BK, BV, 2, D>(a, cbk, cbv, sm, n_ctas, stream);
}

}  // namespace

// All bit-width pairs for head dimension D (instantiated once per D, each in
// its own translation unit: attend_d64.cu, attend_d128.cu, attend_d256.cu).
template <int D>
cudaError_t launch_attend_d(const AttendArgs& a, const Codebook& cbk, const Codebook& cbv,
                            const SignMask& sm, int n_ctas, cudaStream_t stream) {
#ifdef TQ_TEST_INJECT_WAIT_FAULTS
  // the wait test build holds K4/V2 only
  if (a.bits_k * 8 + a.bits_v != 4 * 8 + 2) return cudaErrorNotSupported;
  return launch_pair<4, 2, D>(a, cbk, cbv, sm, n_ctas, stream);
#else
  switch (a.bits_k * 8 + a.bits_v) {
    case 4 * 8 + 2: return launch_pair<4, 2, D>(a, cbk, cbv, sm, n_ctas, stream);
    case 3 * 8 + 2: return launch_pair<3, 2, D>(a, cbk, cbv, sm, n_ctas, stream);
    case 4 * 8 + 3: return launch_pair<4, 3, D>(a, cbk, cbv, sm, n_ctas, stream);
    case 2 * 8 + 2: return launch_pair<2, 2, D>(a, cbk, cbv, sm, n_ctas, stream);
    case 3 * 8 + 3: return launch_pair<3, 3, D>(a, cbk, cbv, sm, n_ctas, stream);
    case 4 * 8 + 4: return launch_pair<4, 4, D>(a, cbk, cbv, sm, n_ctas, stream);
    case 2 * 8 + 3: return launch_pair<2, 3, D>(a, cbk, cbv, sm, n_ctas, stream);
    case 2 * 8 + 4: return launch_pair<2, 4, D>(a, cbk, cbv, sm, n_ctas, stream);
    case 3 * 8 + 4: return launch_pair<3, 4, D>(a, cbk, cbv, sm, n_ctas, stream);
    default: return cudaErrorInvalidValue;
  }
#endif
}

}  // namespace tq
