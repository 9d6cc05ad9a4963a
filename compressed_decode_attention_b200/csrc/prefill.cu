// tq_prefill_attend on the B200 tensor cores (tcgen05, TMEM): causal
// attention of a chunk of T new query tokens over the compressed cache.
//
// [TQPLUS §3] reports prefill speed with the compressed cache; the scores
// and the weighted sum are those of decode ([ADAPTQ §How it works, item 3]:
// rotated query, codebook values of the packed indices, inverse rotation of
// the output). With 128 query rows per kv head and chunk this is a dense
// contraction, so each 128-position chunk of the cache is dequantized once
// into shared-memory operand tiles and reused by all rows.
//
// One CTA per (context split, sequence, kv head, tile of 128 query rows); a
// row is a (token, query head of the GQA group) pair. Warp roles:
//   warps 0-3   one thread per row: rotate its query (thread-local FWHT)
//               into fp16 high/low parts in tensor memory; per chunk two
//               passes over the row of scores (32-column loads, two per
//               wait): the first scales them by the K norms, masks them
//               causally, writes them back and takes the maximum; the
//               second takes the weights (online softmax in the log2
//               domain; the output row is rescaled when the reference
//               maximum moves) and writes the row of P' = weight x V norm
//               (fp16 pairs) over the columns of its own scores; at the end
//               read the output row, normalize, inverse-rotate and store it
//               (or the split's record)
//   warps 4-7   dequantize K: codebook values as fp16 high and low tiles
//               [128 positions x 128 coordinates], and the chunk's norms
//   warps 8-9   dequantize V [128 positions x 128 coordinates]
//   warp 10     bulk copies of the packed rows and norms (two K slots and
//               two V slots)
//   warp 11     tensor memory (512 columns: two 128-column score buffers,
//               the 128-column output, the query's high and low parts); one
//               thread issues per chunk
//                 S = Q_hi·K_hi + Q_lo·K_hi + Q_hi·K_lo  (M 128, N 128, K 128)
//                 O += P'·V                              (M 128, N 128, K 128)
//               kind::f16 MMAs with fp32 accumulators, the A operands (Q,
//               P') in tensor memory, scores one chunk ahead of P'·V
// K tiles are K-major and the V tile MN-major (position rows of
// coordinates), in the 128-byte swizzle layout (tc_common.cuh). K tiles are
// double-buffered (a buffer is free once its scores are done), the V tile
// is single (free once its P'·V is done), and a score buffer is reused
// once the P'·V that read its P' is done.
// The high/low split keeps ~22 significant bits of the scores as in decode;
// P' and V are fp16 as in decode. Every wait is bounded; a role that gives
// up sets TQ_DEV_WAIT_TIMEOUT and stops, and the tensor memory is freed
// after a CTA barrier on every path.
#include <atomic>

#include "attend_kernel.cuh"
#include "tc_common.cuh"

namespace tq {
namespace {

constexpr int kTRows = 128;                       // query rows per tile (MMA M)
constexpr int kTChunk = 128;                      // cache positions per chunk (MMA N)
constexpr int kTD = 128;                          // head dimension
constexpr int kTWarps = 12;
constexpr int kTThreads = 32 * kTWarps;
constexpr int kTNormSlots = 4;                    // ring of per-chunk norms
constexpr long long kTWait = 2000000000LL;         // cycles (~1 s)
// tensor-memory columns
constexpr uint32_t kColS = 0;                     // 2 x 128: scores, then P' (fp16 pairs)
constexpr uint32_t kColO = 256;                   // 128: output accumulator
constexpr uint32_t kColQH = 384, kColQL = 448;    // 64 each: query parts (fp16 pairs)
constexpr uint32_t kTTmemCols = 512;

template <int BK, int BV>
struct TcGeo {
  static constexpr int RK = 16 * BK, RV = 16 * BV;            // packed row bytes (d = 128)
  static constexpr int TILE = kTChunk * kTD * 2;              // 32 KB: [128 x 128] fp16
  static constexpr int KH = 0;                                // 2 K high tiles
  static constexpr int KL = KH + 2 * TILE;                    // 2 K low tiles
  static constexpr int VV = KL + 2 * TILE;                    // the V tile
  // staging: K slots (packed K rows, then the K and V norms) and V slots
  static constexpr int KSLOT = kTChunk * RK + 2 * kTChunk * 2, VSLOT = kTChunk * RV;
  static constexpr int STG = VV + TILE;                       // 2 staging slots
  static constexpr int VSTG = STG + 2 * KSLOT;
  static constexpr int NKF = VSTG + 2 * VSLOT;                // norm ring: 128 floats a slot
  static constexpr int NVF = NKF + kTNormSlots * kTChunk * 4;
  // codebook tables, several copies where a warp's random lookups would
  // collide in shared-memory banks (lane l reads copy l % KREP): K (uint2
  // per pair code) 16 copies where they fit (conflict-free: a 64-bit load
  // serves 16 lanes at a time), else 8, 1 at 2 bits; V (uint32 per pair
  // code) 8 copies unless 2-bit
  static constexpr int LUTK = NVF + kTNormSlots * kTChunk * 4;
  static constexpr int VREP = BV == 2 ? 1 : 8;
  static constexpr bool K16 = LUTK + (1 << (2 * BK)) * 8 * 16 + (1 << (2 * BV)) * 4 * VREP +
                              20 * 8 + 16 + 1024 <= 227 * 1024;
  static constexpr int KREP = BK == 2 ? 1 : K16 ? 16 : 8;
  static constexpr int KSH = BK == 2 ? 3 : K16 ? 7 : 6, VSH = BV == 2 ? 2 : 5;  // log2 bytes per code
  static constexpr int LUTV = LUTK + (1 << (2 * BK)) * 8 * KREP;
  static constexpr int BARS = LUTV + (1 << (2 * BV)) * 4 * VREP;  // 20 barriers
  static constexpr int MISC = BARS + 20 * 8;                  // TMEM address, abort flag
  static constexpr int SMEM = 1024 + MISC + 16;
  static_assert(KSLOT % 16 == 0 && VSLOT % 16 == 0 && STG % 1024 == 0 && NKF % 16 == 0 && BARS % 8 == 0, "align");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int BK, int BV>
__global__ void __launch_bounds__(kTThreads, 1)
prefill_tc_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ Codebook cbk,
                  const __grid_constant__ Codebook cbv, const __grid_constant__ SignMask sm) {
  using G = TcGeo<BK, BV>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::saddr(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sb - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int GQ = a.gqa, H = a.n_kv_heads, T = a.n_tok;
  const int TQ = kTRows / GQ;                      // query tokens per tile
  const int tiles = (T + TQ - 1) / TQ;
  const int S = a.n_splits > 1 ? a.n_splits : 1;
  const int split = blockIdx.x % S;
  const int unit = blockIdx.x / S;
  const int tile = unit % tiles;
  const int g = (unit / tiles) % H;
  const int b = unit / (tiles * H);
  const int i0 = tile * TQ, nq = min(TQ, T - i0);
  const int R = nq * GQ;                           // valid rows
  // barriers (chunk c uses slot c & 1 of the two-deep rings, c & 3 of the
  // four-deep one): staging full/free, K ready (x4), V ready (x1), scores
  // full, P' ready, P'·V done, query ready
  const uint32_t bars = sb + G::BARS;
  auto kst_full = [&](int c) { return bars + 8 * (0 + (c & 1)); };
  auto kst_free = [&](int c) { return bars + 8 * (2 + (c & 1)); };
  auto vst_full = [&](int c) { return bars + 8 * (16 + (c & 1)); };
  auto vst_free = [&](int c) { return bars + 8 * (18 + (c & 1)); };
  auto k_ready = [&](int c) { return bars + 8 * (4 + (c & 3)); };
  const uint32_t v_ready = bars + 8 * 8;
  auto s_full = [&](int c) { return bars + 8 * (9 + (c & 1)); };
  auto p_ready = [&](int c) { return bars + 8 * (11 + (c & 1)); };
  auto pv_done = [&](int c) { return bars + 8 * (13 + (c & 1)); };
  const uint32_t q_ready = bars + 8 * 15;
  // phase parity of chunk c's use of a one-, two- or four-deep ring slot
  auto par1 = [](int c) { return (uint32_t)(c & 1); };
  auto par2 = [](int c) { return (uint32_t)((c >> 1) & 1); };
  auto par4 = [](int c) { return (uint32_t)((c >> 2) & 1); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + G::MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + G::MISC + 4);
  auto wait = [&](uint32_t bar, uint32_t parity) {
    if (*reinterpret_cast<volatile int*>(abort_flag)) return false;
    if (tc::bar_wait(bar, parity, kTWait)) return true;
    atomicExch(abort_flag, 1);
    return false;
  };

  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // ---- codebook tables (launch parameters): K high/low pairs, V pairs
  for (int code = tid; code < (1 << (2 * BK)); code += kTThreads) {
    uint32_t hl[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float c = cbk.centroid[e == 0 ? code & ((1 << BK) - 1) : code >> BK] * kKScale;
      const __half h = __float2half_rn(c), l = __float2half_rn(c - __half2float(h));
      hl[e] = (uint32_t)__half_as_ushort(h) | ((uint32_t)__half_as_ushort(l) << 16);
    }
    const uint2 e = make_uint2((hl[0] & 0xFFFFu) | (hl[1] << 16), (hl[0] >> 16) | (hl[1] & 0xFFFF0000u));
#pragma unroll 1
    for (int rep = 0; rep < G::KREP; ++rep)
      *reinterpret_cast<uint2*>(smem + G::LUTK + (code << G::KSH) + 8 * rep) = e;
  }
  for (int code = tid; code < (1 << (2 * BV)); code += kTThreads) {
    const uint32_t v0 = __half_as_ushort(__float2half_rn(cbv.centroid[code & ((1 << BV) - 1)]));
    const uint32_t v1 = __half_as_ushort(__float2half_rn(cbv.centroid[code >> BV]));
#pragma unroll 1
    for (int rep = 0; rep < G::VREP; ++rep)
      *reinterpret_cast<uint32_t*>(smem + G::LUTV + (code << G::VSH) + 4 * rep) = v0 | (v1 << 16);
  }
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::bar_init(kst_full(i), 1);
      tc::bar_init(kst_free(i), 4);                // the K-dequantizing warps
      tc::bar_init(vst_full(i), 1);
      tc::bar_init(vst_free(i), 2);                // the V-dequantizing warps
      tc::bar_init(s_full(i), 1);
      tc::bar_init(p_ready(i), 4);
      tc::bar_init(pv_done(i), 1);
    }
    for (int i = 0; i < 4; ++i) tc::bar_init(k_ready(i), 4);
    tc::bar_init(v_ready, 2);
    tc::bar_init(q_ready, 4);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 11) tc::tmem_alloc(tc::saddr(tmem_slot), kTTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int raw_len = a.ctx_lens[b];
  const int L = min(max(raw_len, 0), a.cap_tok);
  const int start = L - T;                         // absolute position of token 0
  if (tile == 0 && g == 0 && split == 0 && tid == 0 && a.dev_status) {
    if (raw_len > a.cap_tok) atomicOr(a.dev_status, TQ_DEV_CTX_CLAMPED);
    if (L < T) atomicOr(a.dev_status, TQ_DEV_CTX_EMPTY);
  }
  const int p_last = start + i0 + nq - 1;          // last query position of the tile
  const int nch_tile = p_last >= 0 ? p_last / kTChunk + 1 : 0;
  const int cbase = (int)((long long)split * nch_tile / S);
  const int nchunks = (int)((long long)(split + 1) * nch_tile / S) - cbase;
  const size_t seq_row = ((size_t)b * H + g) * a.cap_tok;

  if (warp == 10) {
    // ---- producer: lane 0 copies chunk c's K rows and norms into K slot
    // c & 1, lane 1 its V rows into V slot c & 1 (each side runs ahead of
    // the other as far as its own slots allow)
    if (lane < 2) {
      const bool kside = lane == 0;
      int c = 0;
      for (; c < nchunks; ++c) {
        if (!wait(kside ? kst_free(c) : vst_free(c), par2(c) ^ 1)) break;
        const int t0 = (cbase + c) * kTChunk;
        const int rows = min(kTChunk, L - t0);
        const int nrows = min(kTChunk, (rows + 7) & ~7);
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        // the rows lie in the sequence's capacity (checked in the
        // bounds-checked build; a skipped copy still completes the phase)
        const bool inb = tq_check(t0 >= 0 && rows > 0 && t0 + nrows <= a.cap_tok, a.dev_status);
        if (kside) {
          const uint32_t dst = sb + G::STG + (c & 1) * G::KSLOT;
          tc::bar_expect(kst_full(c), inb ? rows * G::RK + 4 * nrows : 0u);
          if (inb) {
            tc::bulk_g2s(dst, a.packed_k + (seq_row + t0) * G::RK, rows * G::RK, kst_full(c));
            tc::bulk_g2s(dst + kTChunk * G::RK, a.norms_k + seq_row + t0, 2 * nrows, kst_full(c));
            tc::bulk_g2s(dst + kTChunk * G::RK + 2 * kTChunk, a.norms_v + seq_row + t0, 2 * nrows,
                         kst_full(c));
          }
        } else {
          const uint32_t dst = sb + G::VSTG + (c & 1) * G::VSLOT;
          tc::bar_expect(vst_full(c), inb ? rows * G::RV : 0u);
          if (inb)
            tc::bulk_g2s(dst, a.packed_v + (seq_row + t0) * G::RV, rows * G::RV, vst_full(c));
        }
      }
      // copies still in flight complete before the CTA can end
      for (int k = c > 2 ? c - 2 : 0; k < c; ++k)
        tc::bar_wait(kside ? kst_full(k) : vst_full(k), par2(k), kTWait);
    }
  } else if (warp == 11) {
    // ---- MMA issue (one thread)
    if (lane == 0) {
      constexpr uint32_t idS = tc::umma_idesc(0u, kTRows, kTChunk);
      constexpr uint32_t idO = tc::umma_idesc(0u, kTRows, kTD) | (1u << 16);  // B MN-major
      bool ok = nchunks == 0 || wait(q_ready, 0);
      uint32_t last_bar = 0, last_par = 0;        // the latest commit's barrier and phase
      // descriptors of buffer 0, k-step 0 (a start address moves the low
      // field by bytes / 16)
      const uint64_t kdesc = tc::umma_desc(sb + G::KH);
      const uint64_t vdesc = tc::umma_desc_mn(sb + G::VV, kTChunk * 128, 1024);
      auto scores = [&](int c) {
        // K buffer c & 1 ready; score buffer c & 1 free once the P'·V of
        // chunk c - 2 (which read its P') is done
        if (!wait(k_ready(c), par4(c)) || (c >= 2 && !wait(pv_done(c - 2), par2(c - 2))))
          return false;
        tc::fence_after_sync();
        const uint32_t d = tmem + kColS + kTChunk * (c & 1);
        const uint64_t kb = kdesc + (uint32_t)(((c & 1) * G::TILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTD / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * (kTChunk * 128) + (kk & 3) * 32;
          const uint64_t kh = kb + (koff >> 4);
          const uint64_t kl = kb + ((koff + (G::KL - G::KH)) >> 4);
          tc::mma_f16_ts(d, tmem + kColQH + 8 * kk, kh, idS, kk > 0);
          tc::mma_f16_ts(d, tmem + kColQL + 8 * kk, kh, idS, true);
          tc::mma_f16_ts(d, tmem + kColQH + 8 * kk, kl, idS, true);
        }
        tc::mma_commit(s_full(c));
        last_bar = s_full(c);
        last_par = par2(c);
        return true;
      };
      auto pv = [&](int c) {
        if (!wait(v_ready, par1(c)) || !wait(p_ready(c), par2(c))) return false;
        tc::fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < kTChunk / 16; ++kk)
          tc::mma_f16_ts(tmem + kColO, tmem + kColS + kTChunk * (c & 1) + 8 * kk,
                         vdesc + (uint32_t)(kk * 2048 >> 4), idO, c > 0 || kk > 0);
        tc::mma_commit(pv_done(c));
        last_bar = pv_done(c);
        last_par = par2(c);
        return true;
      };
      if (ok && nchunks > 0) ok = scores(0);
      for (int c = 0; ok && c < nchunks; ++c) {
        if (c + 1 < nchunks && !scores(c + 1)) break;
        if (!pv(c)) break;
      }
      // the last committed products (and all before them) complete before
      // the tensor memory is freed
      if (last_bar) tc::bar_wait(last_bar, last_par, kTWait);
    }
  } else if (warp >= 8) {
    // ---- V dequantization (warps 8-9, thread v): positions (v & 31) + 32j,
    // coordinates 64·(v >> 5) .. + 63 (eight consecutive positions per
    // quarter warp: the 16-byte tile stores fall in distinct banks)
    const int v = tid - 256;
    const int half = v >> 5;
    const uint32_t vrep = G::VREP > 1 ? 4 * (lane & 7) : 0;   // this lane's table copy
    for (int c = 0; c < nchunks; ++c) {
      // the V tile is free once the P'·V of chunk c - 1 is done
      const bool ok = wait(vst_full(c), par2(c)) && (c == 0 || wait(pv_done(c - 1), par2(c - 1)));
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const uint8_t* st = smem + G::VSTG + (c & 1) * G::VSLOT;
      uint8_t* vp = smem + G::VV;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        const int pos = (v & 31) + 32 * j;
        uint32_t vw[(8 * BV + 3) / 4 + 1];
        load_chunk<8 * BV>(st, pos * G::RV + 8 * BV * half, vw);
        // every table load of the unit before its stores (a store would
        // otherwise hold back the loads that follow it)
        uint32_t p[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          p[e] = lds<uint32_t>(smem, G::LUTV + (pair_code_shifted<BV, G::VSH>(vw, e) | vrep));
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
          *reinterpret_cast<uint4*>(vp + tc::sw128_offset(kTChunk, pos, 64 * half + 8 * jj)) =
              make_uint4(p[4 * jj], p[4 * jj + 1], p[4 * jj + 2], p[4 * jj + 3]);
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        tc::bar_arrive(v_ready);
        tc::bar_arrive(vst_free(c));
      }
    }
  } else if (warp >= 4) {
    // ---- K dequantization (warps 4-7, thread u): positions (u & 63) + 64j,
    // coordinates 64·(u >> 6) .. + 63, and the norms of position u
    const int u = tid - 128;
    const int half = u >> 6;
    const uint32_t krep = 8 * (lane & (G::KREP - 1));        // this lane's table copy
    for (int c = 0; c < nchunks; ++c) {
      const int i = c & 1;
      // K buffer i: free once the scores of chunk c - 2 are done
      const bool ok = wait(kst_full(c), par2(c)) && wait(s_full(c), par2(c) ^ 1);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const uint8_t* st = smem + G::STG + i * G::KSLOT;
      uint8_t* khp = smem + G::KH + i * G::TILE;
      uint8_t* klp = smem + G::KL + i * G::TILE;
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        const int pos = (u & 63) + 64 * j;
        uint32_t kw[(8 * BK + 3) / 4 + 1];
        load_chunk<8 * BK>(st, pos * G::RK + 8 * BK * half, kw);
        // every table load of the unit before its stores
        uint2 p[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          p[e] = lds<uint2>(smem, G::LUTK + (pair_code_shifted<BK, G::KSH>(kw, e) | krep));
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {              // 16-byte chunks: 4 pairs
          const uint32_t off = tc::sw128_offset(kTChunk, pos, 64 * half + 8 * jj);
          *reinterpret_cast<uint4*>(khp + off) =
              make_uint4(p[4 * jj].x, p[4 * jj + 1].x, p[4 * jj + 2].x, p[4 * jj + 3].x);
          *reinterpret_cast<uint4*>(klp + off) =
              make_uint4(p[4 * jj].y, p[4 * jj + 1].y, p[4 * jj + 2].y, p[4 * jj + 3].y);
        }
      }
      {
        // norms as floats; 0 past the sequence end (the copied norm runs
        // stop at a multiple of 8 positions: the rest of the slot is stale)
        const bool live = (cbase + c) * kTChunk + u < L;
        const uint16_t* ns = reinterpret_cast<const uint16_t*>(st + kTChunk * G::RK);
        const int slot = (c & (kTNormSlots - 1)) * kTChunk + u;
        reinterpret_cast<float*>(smem + G::NKF)[slot] =
            live ? __half2float(__ushort_as_half(ns[u])) : 0.f;
        reinterpret_cast<float*>(smem + G::NVF)[slot] =
            live ? __half2float(__ushort_as_half(ns[kTChunk + u])) : 0.f;
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        tc::bar_arrive(k_ready(c));
        tc::bar_arrive(kst_free(c));
      }
    }
  } else {
    // ---- warps 0-3: thread r = row r of the tile (TMEM lane r)
    const int r = tid;
    const bool live_row = r < R;
    const int t = r / GQ, h = r - t * GQ;
    const uint32_t trow = (uint32_t)(32 * warp) << 16;
    float si;
    {
      // rotated query: q~ = H·(D⊙q)·log2(e)/d^{3/2}, scaled by a power of two
      // qs that puts its largest value near 2^14, as fp16 high and low parts
      float x[kTD];
      if (live_row) {
        const size_t qo = (((size_t)b * T + i0 + t) * a.n_q_heads + (size_t)g * GQ + h) * kTD;
        if (a.q_dtype == TQ_F32) {
          const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.q) + qo);
#pragma unroll
          for (int k = 0; k < kTD / 4; ++k) {
            const float4 v = src[k];
            x[4 * k] = v.x; x[4 * k + 1] = v.y; x[4 * k + 2] = v.z; x[4 * k + 3] = v.w;
          }
        } else {
          const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.q) + qo);
          const bool bf = a.q_dtype == TQ_BF16;
#pragma unroll
          for (int k = 0; k < kTD / 8; ++k) {
            const uint4 v = src[k];
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = unpack16x2(w4[e], bf);
              x[8 * k + 2 * e] = f.x;
              x[8 * k + 2 * e + 1] = f.y;
            }
          }
        }
#pragma unroll
        for (int k = 0; k < kTD; ++k) x[k] = apply_sign(x[k], sm.w[k >> 5], k & 31);
#pragma unroll
        for (int s = 1; s < kTD; s <<= 1)
#pragma unroll
          for (int k = 0; k < kTD; ++k)
            if (!(k & s)) {
              const float p = x[k], q = x[k + s];
              x[k] = p + q;
              x[k + s] = p - q;
            }
      } else {
#pragma unroll
        for (int k = 0; k < kTD; ++k) x[k] = 0.f;
      }
      float amax = 0.f;
#pragma unroll
      for (int k = 0; k < kTD; ++k) {
        x[k] *= kLog2e / (128.0f * 11.3137084989847603904f);
        amax = fmaxf(amax, fabsf(x[k]));
      }
      const int e = amax > 0.f ? ilogbf(amax) : 0;
      const float qs = ldexpf(1.f, min(14 - e, 120));
      // 16 columns (32 coordinates) of each part per store
#pragma unroll
      for (int blk = 0; blk < kTD / 32; ++blk) {
        uint32_t hw[16], lw[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float v0 = x[32 * blk + 2 * k] * qs, v1 = x[32 * blk + 2 * k + 1] * qs;
          const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
          hw[k] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
          lw[k] = pack_half2(v0 - __half2float(h0), v1 - __half2float(h1));
        }
        tc::tmem_st16_nowait(tmem + trow + kColQH + 16 * blk, hw);
        tc::tmem_st16_nowait(tmem + trow + kColQL + 16 * blk, lw);
      }
      tc::tmem_wait_st();
      si = live_row ? 1.f / (qs * kKScale) : 1.f;
    }
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) tc::bar_arrive(q_ready);

    const int lim = live_row ? start + i0 + t : -1;  // last visible position
    const float2 si2 = make_float2(si, si);
    // mu: reference maximum of the unscaled scores (score x K norm). It moves
    // only when a row's maximum exceeds it by more than 8 in the base-2
    // exponent, so the output is rarely rescaled; weights are taken as
    // 2^(si·(v - mu) - 8) <= 1 (the factor cancels in O / l), which keeps P'
    // within the V norm's range as in decode
    float mu = -INFINITY, l = 0.f;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      // the scores, and (acquired from the K-dequantizing warps directly)
      // the chunk's norms
      ok = wait(s_full(c), par2(c)) && wait(k_ready(c), par4(c));
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const int t0 = (cbase + c) * kTChunk;
      const int ns = (c & (kTNormSlots - 1)) * kTChunk;
      const float4* nk4 = reinterpret_cast<const float4*>(smem + G::NKF) + ns / 4;
      const float4* nv4 = reinterpret_cast<const float4*>(smem + G::NVF) + ns / 4;
      const uint32_t sbuf = tmem + trow + kColS + kTChunk * (c & 1);
      const bool masked = t0 + kTChunk - 1 > lim;
      // v = score x K norm, -inf past the row's last visible position
      auto scaled = [&](const float (&z)[32], int q, int k, float2& v0, float2& v1) {
        const float4 n = nk4[8 * q + k / 4];
        v0 = __fmul2_rn(make_float2(z[k], z[k + 1]), make_float2(n.x, n.y));
        v1 = __fmul2_rn(make_float2(z[k + 2], z[k + 3]), make_float2(n.z, n.w));
        if (masked) {
          const int p = t0 + 32 * q + k;
          if (p > lim) v0.x = -INFINITY;
          if (p + 1 > lim) v0.y = -INFINITY;
          if (p + 2 > lim) v1.x = -INFINITY;
          if (p + 3 > lim) v1.y = -INFINITY;
        }
      };
      // pass 1: v = score x K norm (masked) written back over the scores,
      // and the chunk's maximum (pieces loaded two at a time: one wait for
      // both)
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll 1
      for (int qp = 0; qp < kTChunk / 64; ++qp) {
        float za[32], zb[32];
        tc::tmem_ld32x2(sbuf + 64 * qp, sbuf + 64 * qp + 32, za, zb);
        uint32_t va[32], vb[32];
#pragma unroll
        for (int k = 0; k < 32; k += 4) {
          float2 v0, v1, v2, v3;
          scaled(za, 2 * qp, k, v0, v1);
          scaled(zb, 2 * qp + 1, k, v2, v3);
          mx0 = fmaxf(mx0, fmaxf(fmaxf(v0.x, v0.y), fmaxf(v1.x, v1.y)));
          mx1 = fmaxf(mx1, fmaxf(fmaxf(v2.x, v2.y), fmaxf(v3.x, v3.y)));
          va[k] = __float_as_uint(v0.x); va[k + 1] = __float_as_uint(v0.y);
          va[k + 2] = __float_as_uint(v1.x); va[k + 3] = __float_as_uint(v1.y);
          vb[k] = __float_as_uint(v2.x); vb[k + 1] = __float_as_uint(v2.y);
          vb[k + 2] = __float_as_uint(v3.x); vb[k + 3] = __float_as_uint(v3.y);
        }
        tc::tmem_st32_nowait(sbuf + 64 * qp, va);
        tc::tmem_st32_nowait(sbuf + 64 * qp + 32, vb);
      }
      tc::tmem_wait_st();
      const float mx = fmaxf(mx0, mx1);
      const float mn = fmaxf(mu, mx);
      // the output row holds earlier chunks' products: rescale it (after the
      // previous P'·V completes) when the reference maximum moves
      const bool grow = mu != -INFINITY && si * (mn - mu) > 8.f;
      const float al = grow ? fast_exp2(si * (mu - mn)) : 1.f;
      if (__any_sync(0xFFFFFFFFu, grow)) {
        ok = wait(pv_done(c - 1), par2(c - 1));
        if (!__all_sync(0xFFFFFFFFu, ok)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
#pragma unroll 1
        for (int q4 = 0; q4 < kTD / 32; ++q4) {
          float z[32];
          tc::tmem_ld32(tmem + trow + kColO + 32 * q4, z);
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float2 y = __fmul2_rn(make_float2(z[k], z[k + 1]), make_float2(al, al));
            z[k] = y.x;
            z[k + 1] = y.y;
          }
          tc::tmem_st32(tmem + trow + kColO + 32 * q4, z);
        }
      }
      if (grow || mu == -INFINITY) mu = mn;
      // pass 2: weights 2^(si·v - si·mu - 8) (0 for masked scores), their
      // sum, and P' over the columns already read: the 16 P' columns of
      // piece q lie in columns 16q .. 16q + 15 of the buffer
      const float off = mu == -INFINITY ? 0.f : -fmaf(si, mu, 8.f);
      const float2 off2 = make_float2(off, off);
      float2 ls = make_float2(0.f, 0.f);
#pragma unroll 1
      for (int qp = 0; qp < kTChunk / 64; ++qp) {
        float z[2][32];
        tc::tmem_ld32x2(sbuf + 64 * qp, sbuf + 64 * qp + 32, z[0], z[1]);
        uint32_t pw[2][16];
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          const int q = 2 * qp + hq;
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            // v, as pass 1 left it
            const float2 v0 = make_float2(z[hq][k], z[hq][k + 1]);
            const float2 v1 = make_float2(z[hq][k + 2], z[hq][k + 3]);
            const float4 n = nv4[8 * q + k / 4];
            const float2 e0 = __ffma2_rn(v0, si2, off2);
            const float2 e1 = __ffma2_rn(v1, si2, off2);
            const float2 w0 = make_float2(fast_exp2(e0.x), fast_exp2(e0.y));
            const float2 w1 = make_float2(fast_exp2(e1.x), fast_exp2(e1.y));
            ls = __fadd2_rn(ls, __fadd2_rn(w0, w1));
            const float2 p0 = __fmul2_rn(w0, make_float2(n.x, n.y));
            const float2 p1 = __fmul2_rn(w1, make_float2(n.z, n.w));
            pw[hq][k / 2] = pack_half2(p0.x, p0.y);
            pw[hq][k / 2 + 1] = pack_half2(p1.x, p1.y);
          }
        }
        // both pieces read: P' of piece q to columns 16q .. 16q + 15
        tc::tmem_st16_nowait(sbuf + 32 * qp, pw[0]);
        tc::tmem_st16_nowait(sbuf + 32 * qp + 16, pw[1]);
      }
      tc::tmem_wait_st();
      l = l * al + (ls.x + ls.y);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::bar_arrive(p_ready(c));
    }

    // ---- output row: acc = O / l, inverse rotation D⊙(H·acc)/d (or the record)
    if (ok && nchunks > 0) {
      ok = wait(pv_done(nchunks - 1), par2(nchunks - 1));
      ok = __all_sync(0xFFFFFFFFu, ok);
    }
    if (ok) {
      float x[kTD];
      if (nchunks > 0) {
        tc::fence_after_sync();
#pragma unroll
        for (int q4 = 0; q4 < kTD / 32; ++q4) {
          float z[32];
          tc::tmem_ld32(tmem + trow + kColO + 32 * q4, z);
#pragma unroll
          for (int k = 0; k < 32; ++k) x[32 * q4 + k] = z[k];
        }
      } else {
#pragma unroll
        for (int k = 0; k < kTD; ++k) x[k] = 0.f;
      }
      if (live_row && S > 1) {
        // records of this split: the unnormalized value sum (rotated
        // domain), the base-2 reference maximum of its weights and their
        // sum (empty: 0, -inf, 0)
        const size_t rec = (size_t)split * ((size_t)a.batch * T * a.n_q_heads) +
                           ((size_t)b * T + i0 + t) * a.n_q_heads + (size_t)g * GQ + h;
        float* dst = a.records + rec * (kTD + 2);
        const bool empty = mu == -INFINITY;
#pragma unroll
        for (int k = 0; k < kTD; k += 2)
          *reinterpret_cast<float2*>(dst + k) =
              make_float2(empty ? 0.f : x[k], empty ? 0.f : x[k + 1]);
        *reinterpret_cast<float2*>(dst + kTD) =
            make_float2(empty ? -INFINITY : fmaf(si, mu, 8.f), empty ? 0.f : l);
      } else if (live_row) {
        const float il = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int k = 0; k < kTD; ++k) x[k] *= il;
#pragma unroll
        for (int s = 1; s < kTD; s <<= 1)
#pragma unroll
          for (int k = 0; k < kTD; ++k)
            if (!(k & s)) {
              const float p = x[k], q = x[k + s];
              x[k] = p + q;
              x[k + s] = p - q;
            }
        const size_t ob = (((size_t)b * T + i0 + t) * a.n_q_heads + (size_t)g * GQ + h) * kTD;
        if (a.out_dtype == TQ_F32) {
          float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + ob);
#pragma unroll
          for (int k = 0; k < kTD; k += 4)
            o[k / 4] = make_float4(apply_sign(x[k], sm.w[k >> 5], k & 31) * (1.f / kTD),
                                   apply_sign(x[k + 1], sm.w[k >> 5], (k + 1) & 31) * (1.f / kTD),
                                   apply_sign(x[k + 2], sm.w[k >> 5], (k + 2) & 31) * (1.f / kTD),
                                   apply_sign(x[k + 3], sm.w[k >> 5], (k + 3) & 31) * (1.f / kTD));
        } else {
          const bool bf = a.out_dtype == TQ_BF16;
          uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.out) + ob);
#pragma unroll
          for (int k = 0; k < kTD; k += 8) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c0 = k + 2 * e;
              const float v0 = apply_sign(x[c0], sm.w[c0 >> 5], c0 & 31) * (1.f / kTD);
              const float v1 = apply_sign(x[c0 + 1], sm.w[c0 >> 5], (c0 + 1) & 31) * (1.f / kTD);
              const uint32_t h0 = bf ? f32_to_bf16_bits(v0) : f32_to_f16_bits(v0);
              const uint32_t h1 = bf ? f32_to_bf16_bits(v1) : f32_to_f16_bits(v1);
              w4[e] = h0 | (h1 << 16);
            }
            o[k / 8] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
    }
  }
  if (tid == 0 && *reinterpret_cast<volatile int*>(abort_flag) && a.dev_status)
    atomicOr(a.dev_status, TQ_DEV_WAIT_TIMEOUT);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 11) tc::tmem_dealloc(tmem, kTTmemCols);
}

template <int BK, int BV>
cudaError_t launch_prefill_bits(const PrefillArgs& a, const Codebook& cbk, const Codebook& cbv,
                                   const SignMask& sm, cudaStream_t stream) {
  using G = TcGeo<BK, BV>;
  static std::atomic<bool> configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<BK, BV>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  const int tq = kTRows / a.gqa;
  const int S = a.n_splits > 1 ? a.n_splits : 1;
  const long long grid = (long long)a.batch * a.n_kv_heads * ((a.n_tok + tq - 1) / tq) * S;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kTThreads);
  cfg.dynamicSmemBytes = G::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_tc_kernel<BK, BV>, a, cbk, cbv, sm);
  if (e != cudaSuccess || S == 1) return e;
  // merge the splits' records and rotate back (the context-parallel combine)
  CombineArgs c;
  c.partials = a.records;
  c.n_parts = S;
  c.n_rec = a.batch * a.n_tok * a.n_q_heads;
  c.d = kTD;
  c.dev_status = a.dev_status;
  c.out = a.out;
  c.out_dtype = a.out_dtype;
  return launch_combine(c, sm, stream);
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, const Codebook& cbk, const Codebook& cbv,
                              const SignMask& sm, cudaStream_t stream) {
  switch (a.bits_k * 8 + a.bits_v) {
    case 4 * 8 + 2: return launch_prefill_bits<4, 2>(a, cbk, cbv, sm, stream);
    case 3 * 8 + 2: return launch_prefill_bits<3, 2>(a, cbk, cbv, sm, stream);
    case 4 * 8 + 3: return launch_prefill_bits<4, 3>(a, cbk, cbv, sm, stream);
    case 2 * 8 + 2: return launch_prefill_bits<2, 2>(a, cbk, cbv, sm, stream);
    case 3 * 8 + 3: return launch_prefill_bits<3, 3>(a, cbk, cbv, sm, stream);
    case 4 * 8 + 4: return launch_prefill_bits<4, 4>(a, cbk, cbv, sm, stream);
    case 2 * 8 + 3: return launch_prefill_bits<2, 3>(a, cbk, cbv, sm, stream);
    case 2 * 8 + 4: return launch_prefill_bits<2, 4>(a, cbk, cbv, sm, stream);
    case 3 * 8 + 4: return launch_prefill_bits<3, 4>(a, cbk, cbv, sm, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tq
