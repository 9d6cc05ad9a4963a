// tq_prefill_attend: causal attention of a chunk of T new query tokens per
// sequence over the compressed cache (the prefill of a chunk whose K/V rows
// were appended with tq_encode), on tensor cores.
//
// [TQPLUS §3] reports prefill speed with the compressed cache; the scores
// and the weighted sum are those of decode ([ADAPTQ §How it works, item 3]:
// rotated query, codebook lookups of the packed indices, inverse rotation of
// the output), per query token with the causal length. With many query rows
// per kv head this is a dense contraction, so unlike decode the cache tile
// is dequantized once into shared memory and reused by every query row.
//
// Decomposition: one CTA per (sequence, kv head, tile of query rows); a row
// is a (token, query head of the GQA group) pair, 16·8 = 128 rows per CTA.
// Per 64-position chunk of the cache:
//   stage    bulk copies of the packed K/V rows and norms (two slots,
//            mbarrier, bounded wait)
//   dequant  all threads: K codebook values as fp16 high/low tiles and V as
//            an fp16 tile, [position][coordinate], 272-byte rows (ldmatrix
//            without bank conflicts)
//   scores   per warp (16 rows): mma.m16n8k16, A = rotated query high/low
//            (registers), B = K tiles (ldmatrix); Q_hi·K_hi + Q_lo·K_hi +
//            Q_hi·K_lo keep ~22 significant bits as in decode
//   softmax  online, fp32, log2 domain, causal mask
//   PV       A = softmax weight x V norm (fp16, from the score registers),
//            B = V tile (ldmatrix.trans)
// Output per row: D⊙(H·(acc/l))/d with in-register and shuffle stages.
#include <atomic>
#include "attend_kernel.cuh"

namespace tq {
namespace {

constexpr int kPfWarps = 8;
constexpr int kPfThreads = 32 * kPfWarps;
constexpr int kPfRows = 16 * kPfWarps;          // query rows per CTA
constexpr int kPfChunk = 64;                    // cache positions per chunk
constexpr int kTS = 136;                        // tile row stride in halves (272 B)

template <int BK, int BV>
struct PfGeo {
  static constexpr int RK = 16 * BK, RV = 16 * BV;          // d = 128
  static constexpr int KROWS = RK % 16 == 0 ? 1 : 16 / (RK % 16);
  static constexpr int VROWS = RV % 16 == 0 ? 1 : 16 / (RV % 16);
  static constexpr int QH = 0;                               // [128 rows][kTS] fp16
  static constexpr int QL = QH + kPfRows * kTS * 2;
  // two buffers of dequantized chunk tiles: K high, K low, V ([64 positions]
  // [kTS] fp16 each) and the K / V norms as floats
  static constexpr int KH = QL + kPfRows * kTS * 2;          // [64 positions][kTS]
  static constexpr int KL = KH + kPfChunk * kTS * 2;
  static constexpr int VT = KL + kPfChunk * kTS * 2;
  static constexpr int NKF = VT + kPfChunk * kTS * 2;        // float [64]
  static constexpr int NVF = NKF + kPfChunk * 4;             // float [64]
  static constexpr int TBUF = NVF + kPfChunk * 4 - KH;       // bytes per buffer
  static constexpr int STG = KH + 2 * TBUF;                  // two staging slots
  static constexpr int SLOT = kPfChunk * (RK + RV) + 2 * kPfChunk * 2;
  static constexpr int LUTK = STG + 2 * SLOT;                // uint2 per pair code
  static constexpr int LUTV = LUTK + (1 << (2 * BK)) * 8;    // uint32 per pair code
  static constexpr int SINV = LUTV + (1 << (2 * BV)) * 4;    // float per row
  static constexpr int MBAR = SINV + kPfRows * 4;
  static constexpr int SMEM = MBAR + 16;
  static_assert(SLOT % 16 == 0 && STG % 16 == 0 && TBUF % 16 == 0 && MBAR % 8 == 0,
                "alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

template <int BK, int BV>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_kernel(const __grid_constant__ PrefillArgs a,
               const __grid_constant__ Codebook cbk,
               const __grid_constant__ Codebook cbv,
               const __grid_constant__ SignMask sm) {
  using G = PfGeo<BK, BV>;
  constexpr int D = 128;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_addr(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int GQ = a.gqa, H = a.n_kv_heads, T = a.n_tok;
  const int TQ = kPfRows / GQ;                     // query tokens per tile
  const int tiles = (T + TQ - 1) / TQ;
  // split s of n_splits takes the s-th share of the tile's chunks and leaves
  // log-sum-exp records for the combine kernel instead of the output
  const int S = a.n_splits > 1 ? a.n_splits : 1;
  const int split = blockIdx.x % S;
  const int unit = blockIdx.x / S;
  const int tile = unit % tiles;
  const int g = (unit / tiles) % H;
  const int b = unit / (tiles * H);
  const int i0 = tile * TQ, nq = min(TQ, T - i0);
  const int R = nq * GQ;                           // valid rows
  float* sinv = reinterpret_cast<float*>(smem + G::SINV);
  const uint32_t bar0 = sbase + G::MBAR;

  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // ---- codebook tables from the launch parameters
  for (int code = tid; code < (1 << (2 * BK)); code += kPfThreads) {
    uint32_t hl[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float c = cbk.centroid[e == 0 ? code & ((1 << BK) - 1) : code >> BK] * kKScale;
      const __half h = __float2half_rn(c), l = __float2half_rn(c - __half2float(h));
      hl[e] = (uint32_t)__half_as_ushort(h) | ((uint32_t)__half_as_ushort(l) << 16);
    }
    *reinterpret_cast<uint2*>(smem + G::LUTK + 8 * code) =
        make_uint2((hl[0] & 0xFFFFu) | (hl[1] << 16), (hl[0] >> 16) | (hl[1] & 0xFFFF0000u));
  }
  for (int code = tid; code < (1 << (2 * BV)); code += kPfThreads) {
    const uint32_t v0 = __half_as_ushort(__float2half_rn(cbv.centroid[code & ((1 << BV) - 1)]));
    const uint32_t v1 = __half_as_ushort(__float2half_rn(cbv.centroid[code >> BV]));
    *reinterpret_cast<uint32_t*>(smem + G::LUTV + 4 * code) = v0 | (v1 << 16);
  }
  if (tid == 0) {
    mbar_init(bar0);
    mbar_init(bar0 + 8);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  asm volatile("griddepcontrol.wait;\n" ::: "memory");

  const int raw = a.ctx_lens[b];
  const int L = min(max(raw, 0), a.cap_tok);
  const int start = L - T;                         // absolute position of token 0
  if (tile == 0 && g == 0 && split == 0 && tid == 0 && a.dev_status) {
    if (raw > a.cap_tok) atomicOr(a.dev_status, TQ_DEV_CTX_CLAMPED);
    if (L < T) atomicOr(a.dev_status, TQ_DEV_CTX_EMPTY);
  }
  const int p_last = start + i0 + nq - 1;          // last query position of the tile
  const int nch_tile = p_last >= 0 ? p_last / kPfChunk + 1 : 0;
  // this CTA's chunks: absolute chunks cbase .. cbase + nchunks - 1 (local
  // index c = 0 .. nchunks - 1 for staging slots and barrier phases)
  const int cbase = (int)((long long)split * nch_tile / S);
  const int nchunks = (int)((long long)(split + 1) * nch_tile / S) - cbase;

  const size_t seq_row = ((size_t)b * H + g) * a.cap_tok;
  auto issue = [&](int c) {                        // thread 0
    const int t0 = (cbase + c) * kPfChunk;
    const int rows = min(kPfChunk, L - t0);
    const int krows = min(kPfChunk, (rows + G::KROWS - 1) / G::KROWS * G::KROWS);
    const int vrows = min(kPfChunk, (rows + G::VROWS - 1) / G::VROWS * G::VROWS);
    const int nrows = min(kPfChunk, (rows + 7) & ~7);
    const uint32_t dst = sbase + G::STG + (c & 1) * G::SLOT, bar = bar0 + 8 * (c & 1);
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    mbar_expect(bar, krows * G::RK + vrows * G::RV + 4 * nrows);
    bulk_g2s(dst, a.packed_k + (seq_row + t0) * G::RK, krows * G::RK, bar);
    bulk_g2s(dst + kPfChunk * G::RK, a.packed_v + (seq_row + t0) * G::RV, vrows * G::RV, bar);
    bulk_g2s(dst + kPfChunk * (G::RK + G::RV), a.norms_k + seq_row + t0, 2 * nrows, bar);
    bulk_g2s(dst + kPfChunk * (G::RK + G::RV) + 2 * kPfChunk, a.norms_v + seq_row + t0,
             2 * nrows, bar);
  };
  if (tid == 0 && nchunks > 0) issue(0);
  if (tid == 0 && nchunks > 1) issue(1);

  // ---- rotated queries: warp w rotates its rows 16w .. 16w + 15 one by one
  // (row r = token r / GQ of the tile, head r % GQ of the group)
  for (int rr = 0; rr < 16; ++rr) {
    const int r = 16 * warp + rr;
    __half* qh = reinterpret_cast<__half*>(smem + G::QH) + r * kTS + 4 * lane;
    __half* ql = reinterpret_cast<__half*>(smem + G::QL) + r * kTS + 4 * lane;
    if (r >= R) {
      *reinterpret_cast<uint2*>(qh) = make_uint2(0u, 0u);
      *reinterpret_cast<uint2*>(ql) = make_uint2(0u, 0u);
      if (lane == 0) sinv[r] = 0.f;
      continue;
    }
    const int t = r / GQ, h = r - t * GQ;
    const size_t qo = (((size_t)b * T + i0 + t) * a.n_q_heads + (size_t)g * GQ + h) * D + 4 * lane;
    float x[4];
    if (a.q_dtype == TQ_F32) {
      const float4 v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.q) + qo);
      x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
      const uint2 v = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(a.q) + qo);
      const bool bf = a.q_dtype == TQ_BF16;
      const float2 f0 = unpack16x2(v.x, bf), f1 = unpack16x2(v.y, bf);
      x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = 4 * lane + k;
      x[k] = apply_sign(x[k], sm.w[c >> 5], c & 31);
    }
    fwht_warp<4>(x, lane);
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
    uint32_t hw[2], lw[2];
#pragma unroll
    for (int k = 0; k < 4; k += 2) {
      const float v0 = x[k] * qs, v1 = x[k + 1] * qs;
      const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
      hw[k / 2] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
      lw[k / 2] = pack_half2(v0 - __half2float(h0), v1 - __half2float(h1));
    }
    *reinterpret_cast<uint2*>(qh) = make_uint2(hw[0], hw[1]);
    *reinterpret_cast<uint2*>(ql) = make_uint2(lw[0], lw[1]);
    if (lane == 0) sinv[r] = 1.f / (qs * kKScale);
  }
  __syncthreads();

  // A fragments of the warp's 16 rows (k-step ks: coordinates 16ks..16ks+15)
  uint32_t qa[8][4], qb[8][4];
  {
    const int row = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
    const int col = 8 * (lane >> 4);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      ldsm_x4(sbase + G::QH + 2 * (row * kTS + 16 * ks + col), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
      ldsm_x4(sbase + G::QL + 2 * (row * kTS + 16 * ks + col), qb[ks][0], qb[ks][1], qb[ks][2], qb[ks][3]);
    }
  }
  const int r0 = 16 * warp + gq, r1 = r0 + 8;      // this lane's rows
  const float si0 = sinv[r0], si1 = sinv[r1];
  const int p0 = r0 < R ? start + i0 + r0 / GQ : -1;   // causal limits (-1: no positions)
  const int p1 = r1 < R ? start + i0 + r1 / GQ : -1;

  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  bool stalled = false;

  // Chunk c: its packed rows arrive in staging slot c & 1 (issued two
  // chunks ahead), are dequantized into tile buffer c & 1, and are consumed
  // by the MMAs of the next round. A warp that finishes the MMAs of chunk c
  // goes on to dequantize chunk c + 1 into the other buffer while the rest
  // still multiply; one barrier per chunk separates the rounds.
  auto dequant = [&](int c) {
    const uint8_t* st = smem + G::STG + (c & 1) * G::SLOT;
    uint8_t* tb = smem + (c & 1) * G::TBUF;        // buffer c & 1 (add G::KH etc.)
    const int pos = tid >> 2, qd = tid & 3;
    uint32_t kw[(4 * BK + 3) / 4 + 1], vw[(4 * BV + 3) / 4 + 1];
    load_chunk<4 * BK>(st, pos * G::RK + 4 * BK * qd, kw);
    load_chunk<4 * BV>(st, kPfChunk * G::RK + pos * G::RV + 4 * BV * qd, vw);
    uint32_t hi[16], lo[16], vv[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      const uint2 e = lds<uint2>(smem, G::LUTK + pair_code_shifted<BK, 3>(kw, p));
      hi[p] = e.x;
      lo[p] = e.y;
      vv[p] = lds<uint32_t>(smem, G::LUTV + pair_code_shifted<BV, 2>(vw, p));
    }
    const int off = 2 * (pos * kTS + 32 * qd);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      *reinterpret_cast<uint4*>(tb + G::KH + off + 16 * k) =
          make_uint4(hi[4 * k], hi[4 * k + 1], hi[4 * k + 2], hi[4 * k + 3]);
      *reinterpret_cast<uint4*>(tb + G::KL + off + 16 * k) =
          make_uint4(lo[4 * k], lo[4 * k + 1], lo[4 * k + 2], lo[4 * k + 3]);
      *reinterpret_cast<uint4*>(tb + G::VT + off + 16 * k) =
          make_uint4(vv[4 * k], vv[4 * k + 1], vv[4 * k + 2], vv[4 * k + 3]);
    }
    if (qd == 0) {
      // norms as floats; 0 past the sequence end (the copied norm runs stop
      // at a multiple of 8 positions: the rest of the slot is stale)
      const bool live = (cbase + c) * kPfChunk + pos < L;
      const uint16_t* nsrc = reinterpret_cast<const uint16_t*>(st + kPfChunk * (G::RK + G::RV));
      reinterpret_cast<float*>(tb + G::NKF)[pos] =
          live ? __half2float(__ushort_as_half(nsrc[pos])) : 0.f;
      reinterpret_cast<float*>(tb + G::NVF)[pos] =
          live ? __half2float(__ushort_as_half(nsrc[kPfChunk + pos])) : 0.f;
    }
  };
  // the first chunk: its data, its tiles, then slot 0 is free for chunk 2
  int issued = nchunks > 0 ? (nchunks > 1 ? 2 : 1) : 0;   // chunks 0, 1 in flight
  if (nchunks > 0) {
    const bool ok = mbar_wait(bar0, 0u);
    if (ok) dequant(0);
    if (!__syncthreads_and(ok)) {                  // the first copy never completed
      stalled = true;
      if (tid == 0) {
        if (a.dev_status) atomicOr(a.dev_status, TQ_DEV_WAIT_TIMEOUT);
        for (int k = 0; k < issued; ++k) mbar_wait(bar0 + 8 * (k & 1), (uint32_t)(k >> 1) & 1u);
      }
    } else {
      if (tid == 0 && nchunks > 2) issue(2);
      issued = min(nchunks, 3);
    }
  }
  for (int c = 0; c < nchunks && !stalled; ++c) {
    const uint8_t* tb = smem + (c & 1) * G::TBUF;
    const uint32_t tbs = sbase + (c & 1) * G::TBUF;
    // ---- scores of the warp's 16 rows x 64 positions
    const int t0 = (cbase + c) * kPfChunk;
    const float* nkf = reinterpret_cast<const float*>(tb + G::NKF);
    const float* nvf = reinterpret_cast<const float*>(tb + G::NVF);
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    {
      // ldmatrix x4: two n-tiles (positions 16 n2 .. + 15) x (coords lo / hi 8)
      const int prow = (lane & 7) + 8 * (lane >> 4), pcol = 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int n2 = 0; n2 < 4; ++n2) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t bh0, bh1, bh2, bh3, bl0, bl1, bl2, bl3;
          const uint32_t o2 = 2 * ((16 * n2 + prow) * kTS + 16 * ks + pcol);
          ldsm_x4(tbs + G::KH + o2, bh0, bh1, bh2, bh3);
          ldsm_x4(tbs + G::KL + o2, bl0, bl1, bl2, bl3);
          mma16816(s[2 * n2], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], bh0, bh1);
          mma16816(s[2 * n2], qb[ks][0], qb[ks][1], qb[ks][2], qb[ks][3], bh0, bh1);
          mma16816(s[2 * n2], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], bl0, bl1);
          mma16816(s[2 * n2 + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], bh2, bh3);
          mma16816(s[2 * n2 + 1], qb[ks][0], qb[ks][1], qb[ks][2], qb[ks][3], bh2, bh3);
          mma16816(s[2 * n2 + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], bl2, bl3);
        }
      }
    }
    // ---- scale, causal mask, online softmax (rows r0: s[.][0..1], r1: [2..3])
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int pl = 8 * nt + 2 * tq + e, pos = t0 + pl;
        const float nk = nkf[pl];
        float v0 = s[nt][e] * (si0 * nk), v1 = s[nt][2 + e] * (si1 * nk);
        if (pos > p0) v0 = -INFINITY;
        if (pos > p1) v1 = -INFINITY;
        s[nt][e] = v0;
        s[nt][2 + e] = v1;
        mx0 = fmaxf(mx0, v0);
        mx1 = fmaxf(mx1, v1);
      }
#pragma unroll
    for (int o2 = 1; o2 <= 2; o2 <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, o2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, o2));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float al0 = mn0 == -INFINITY ? 1.f : fast_exp2(m0 - mn0);
    const float al1 = mn1 == -INFINITY ? 1.f : fast_exp2(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    l0 *= al0;
    l1 *= al1;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      o[j][0] *= al0;
      o[j][1] *= al0;
      o[j][2] *= al1;
      o[j][3] *= al1;
    }
    uint32_t pa[4][4];                              // P' A fragments per 16 positions
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float w[4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int pl = 8 * nt + 2 * tq + e;
        const float nv = nvf[pl];
        const float w0 = s[nt][e] == -INFINITY ? 0.f : fast_exp2(s[nt][e] - mn0);
        const float w1 = s[nt][2 + e] == -INFINITY ? 0.f : fast_exp2(s[nt][2 + e] - mn1);
        l0 += w0;
        l1 += w1;
        w[e] = w0 * nv;
        w[2 + e] = w1 * nv;
      }
      const int kk = nt >> 1, hf = nt & 1;
      pa[kk][2 * hf] = pack_half2(w[0], w[1]);          // row gq
      pa[kk][2 * hf + 1] = pack_half2(w[2], w[3]);      // row gq + 8
    }
    // ---- O += P'·V (k = positions 16kk.., n = coordinates 8j..)
    {
      const int vrow = (lane & 7) + 8 * ((lane >> 3) & 1), vcol = 8 * (lane >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int j2 = 0; j2 < 8; ++j2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(tbs + G::VT + 2 * ((16 * kk + vrow) * kTS + 16 * j2 + vcol), b0, b1, b2, b3);
          mma16816(o[2 * j2], pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3], b0, b1);
          mma16816(o[2 * j2 + 1], pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3], b2, b3);
        }
      }
    }
    // ---- the next chunk into the other buffer (its last readers were the
    // MMAs of chunk c - 1, finished before the previous barrier)
    if (c + 1 < nchunks) {
      const bool ok = mbar_wait(bar0 + 8 * ((c + 1) & 1), (uint32_t)((c + 1) >> 1) & 1u);
      if (ok) dequant(c + 1);
      if (!__syncthreads_and(ok)) {                // a copy never completed
        stalled = true;
        if (tid == 0 && a.dev_status) atomicOr(a.dev_status, TQ_DEV_WAIT_TIMEOUT);
        // wait (bounded) for the copies still in flight, then stop
        if (tid == 0)
          for (int k = c + 1; k < issued; ++k)
            mbar_wait(bar0 + 8 * (k & 1), (uint32_t)(k >> 1) & 1u);
        break;
      }
      // slot (c + 1) & 1 is consumed: chunk c + 3 goes there
      if (tid == 0 && c + 3 < nchunks) issue(c + 3);
      if (c + 3 < nchunks) issued = c + 4;
    }
  }

  // ---- per-row sums, normalization, inverse rotation, store
#pragma unroll
  for (int o2 = 1; o2 <= 2; o2 <<= 1) {
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, o2);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, o2);
  }
  if (S > 1) {
    // records of this split: the unnormalized value sum (rotated domain),
    // the base-2 running maximum and the sum, per row (empty: 0, -inf, 0)
#pragma unroll
    for (int rsel = 0; rsel < 2; ++rsel) {
      const int r = rsel ? r1 : r0;
      if (r >= R) continue;
      const int t = r / GQ, h = r - t * GQ;
      const size_t rec = (size_t)split * ((size_t)a.batch * T * a.n_q_heads) +
                         ((size_t)b * T + i0 + t) * a.n_q_heads + (size_t)g * GQ + h;
      float* dst = a.records + rec * (D + 2);
      const float m = stalled ? -INFINITY : (rsel ? m1 : m0);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float v0 = stalled || m == -INFINITY ? 0.f : o[j][2 * rsel];
        const float v1 = stalled || m == -INFINITY ? 0.f : o[j][2 * rsel + 1];
        *reinterpret_cast<float2*>(dst + 8 * j + 2 * tq) = make_float2(v0, v1);
      }
      if (tq == 0)
        *reinterpret_cast<float2*>(dst + D) =
            make_float2(m, m == -INFINITY ? 0.f : (rsel ? l1 : l0));
    }
    return;
  }
  const float il0 = l0 > 0.f && !stalled ? 1.f / l0 : 0.f;
  const float il1 = l1 > 0.f && !stalled ? 1.f / l1 : 0.f;
  // x[k][e]: coordinate 8k + 2tq + e of row r0 (y: row r1)
  float x[16][2], y[16][2];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    x[j][0] = o[j][0] * il0; x[j][1] = o[j][1] * il0;
    y[j][0] = o[j][2] * il1; y[j][1] = o[j][3] * il1;
  }
  // Walsh-Hadamard over the 128 coordinates c = 8j + 2tq + e: bit 0 in the
  // register pair, bits 1-2 across the four lanes tq, bits 3-6 across j.
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float u = x[j][0], v = x[j][1];
    x[j][0] = u + v; x[j][1] = u - v;
    u = y[j][0]; v = y[j][1];
    y[j][0] = u + v; y[j][1] = u - v;
  }
#pragma unroll
  for (int ob = 1; ob <= 2; ob <<= 1) {
    const bool upper = tq & ob;
#pragma unroll
    for (int j = 0; j < 16; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float px = __shfl_xor_sync(0xFFFFFFFFu, x[j][e], ob);
        const float py = __shfl_xor_sync(0xFFFFFFFFu, y[j][e], ob);
        x[j][e] = upper ? px - x[j][e] : x[j][e] + px;
        y[j][e] = upper ? py - y[j][e] : y[j][e] + py;
      }
  }
#pragma unroll
  for (int sj = 1; sj < 16; sj <<= 1)
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (!(j & sj))
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float u = x[j][e], v = x[j + sj][e];
          x[j][e] = u + v; x[j + sj][e] = u - v;
          u = y[j][e]; v = y[j + sj][e];
          y[j][e] = u + v; y[j + sj][e] = u - v;
        }
#pragma unroll
  for (int rsel = 0; rsel < 2; ++rsel) {
    const int r = rsel ? r1 : r0;
    if (r >= R) continue;
    const int t = r / GQ, h = r - t * GQ;
    const size_t ob = (((size_t)b * T + i0 + t) * a.n_q_heads + (size_t)g * GQ + h) * D;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int c = 8 * j + 2 * tq;
      float v0 = rsel ? y[j][0] : x[j][0], v1 = rsel ? y[j][1] : x[j][1];
      v0 = apply_sign(v0, sm.w[c >> 5], c & 31) * (1.f / D);
      v1 = apply_sign(v1, sm.w[(c + 1) >> 5], (c + 1) & 31) * (1.f / D);
      if (a.out_dtype == TQ_F32) {
        *reinterpret_cast<float2*>(reinterpret_cast<float*>(a.out) + ob + c) = make_float2(v0, v1);
      } else {
        const bool bf = a.out_dtype == TQ_BF16;
        const uint32_t h0 = bf ? f32_to_bf16_bits(v0) : f32_to_f16_bits(v0);
        const uint32_t h1 = bf ? f32_to_bf16_bits(v1) : f32_to_f16_bits(v1);
        *reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(a.out) + ob + c) = h0 | (h1 << 16);
      }
    }
  }
}

template <int BK, int BV>
cudaError_t launch_prefill_bits(const PrefillArgs& a, const Codebook& cbk, const Codebook& cbv,
                                const SignMask& sm, cudaStream_t stream) {
  using G = PfGeo<BK, BV>;
  // set once per device (idempotent; atomic so that concurrent first calls do not race)
  static std::atomic<bool> configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(prefill_kernel<BK, BV>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  const int tq = kPfRows / a.gqa;
  const int S = a.n_splits > 1 ? a.n_splits : 1;
  const long long grid = (long long)a.batch * a.n_kv_heads * ((a.n_tok + tq - 1) / tq) * S;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kPfThreads);
  cfg.dynamicSmemBytes = G::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_kernel<BK, BV>, a, cbk, cbv, sm);
  if (e != cudaSuccess || S == 1) return e;
  // merge the splits' records and rotate back (the context-parallel combine)
  CombineArgs c;
  c.partials = a.records;
  c.n_parts = S;
  c.n_rec = a.batch * a.n_tok * a.n_q_heads;
  c.d = 128;
  c.dev_status = a.dev_status;
  c.out = a.out;
  c.out_dtype = a.out_dtype;
  return launch_combine(c, sm, stream);
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, const Codebook& cbk, const Codebook& cbv,
                           const SignMask& sm, cudaStream_t stream) {
  return launch_prefill_tc(a, cbk, cbv, sm, stream);
}

cudaError_t launch_prefill_mma_sync(const PrefillArgs& a, const Codebook& cbk,
                                    const Codebook& cbv, const SignMask& sm, cudaStream_t stream) {
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
