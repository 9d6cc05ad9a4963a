// C ABI entry points: argument validation on the host, then kernel launches
// on the caller's stream. Declarations and contracts: include/tq.h.
#include <math.h>
#include <stdint.h>

#include "tq.h"
#include "tq_internal.h"

using namespace tq;

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int check_head_dim(int d) {
  if (d <= 0 || (d & (d - 1))) return TQ_ERR_INVALID_ARG;
  if (d < 64 || d > 256) return TQ_ERR_INVALID_ARG;
  return TQ_OK;                              // 64, 128, 256
}

bool bits_ok(int b) { return b >= 2 && b <= 4; }

constexpr int kMaxGridYZ = 65535;   // CUDA grid y/z limit (heads, batch)

int from_cuda(cudaError_t e) { return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA; }

}  // namespace


namespace tq {

// Validation and launch shared by tq_attend, tq_attend_append and
// tq_attend_partial (partial_out: out receives log-sum-exp records).
int attend_common(const void* q, int q_dtype, const void* new_kv, int kv_dtype,
                  uint8_t* packed_k, uint16_t* norms_k, uint8_t* packed_v,
                  uint16_t* norms_v, const int32_t* ctx_lens, int batch, int n_q_heads,
                  int gqa_ratio, int d, int bits_k, int bits_v, uint64_t seed, int cap_tok,
                  float sparse_v_thresh, int n_ctas, void* workspace, size_t workspace_bytes,
                  int* dev_status, unsigned long long* sparse_v_skipped, void* out,
                  int out_dtype, int partial_out, void* stream,
                  unsigned int* head_skipped = nullptr) {
  if (batch < 1 || n_q_heads < 1 || gqa_ratio < 1 || cap_tok < 1)
    return TQ_ERR_INVALID_ARG;
  if (n_q_heads % gqa_ratio) return TQ_ERR_INVALID_ARG;
  if (gqa_ratio > kMaxGroup) return TQ_ERR_UNSUPPORTED;
  if (q_dtype < TQ_F16 || q_dtype > TQ_F32 || out_dtype < TQ_F16 || out_dtype > TQ_F32)
    return TQ_ERR_INVALID_ARG;
  if (!bits_ok(bits_k) || !bits_ok(bits_v)) return TQ_ERR_INVALID_ARG;
  if (n_ctas < 0 || n_ctas > kMaxCtas) return TQ_ERR_INVALID_ARG;
  if (isnan(sparse_v_thresh)) return TQ_ERR_INVALID_ARG;
  const int hd = check_head_dim(d);
  if (hd != TQ_OK) return hd;
  if (cap_tok % 8) return TQ_ERR_UNSUPPORTED;
  if (!q || !packed_k || !norms_k || !packed_v || !norms_v || !ctx_lens || !out ||
      !workspace)
    return TQ_ERR_INVALID_ARG;
  // records (partial_out) are written two floats at a time: 8-byte alignment
  const bool out_ok = partial_out ? ((uintptr_t)out & 7u) == 0 : aligned16(out);
  if (!aligned16(q) || !out_ok || !aligned16(packed_k) || !aligned16(packed_v) ||
      !aligned16(norms_k) || !aligned16(norms_v) || !aligned16(workspace) ||
      ((uintptr_t)ctx_lens & 3u) || ((uintptr_t)sparse_v_skipped & 7u) ||
      ((uintptr_t)dev_status & 3u) || ((uintptr_t)head_skipped & 3u))
    return TQ_ERR_INVALID_ARG;
  if (workspace_bytes < attend_workspace_bytes(batch, n_q_heads, d)) return TQ_ERR_INVALID_ARG;
  const Codebook* cbk = codebook_for(bits_k);
  const Codebook* cbv = codebook_for(bits_v);
  if (!cbk || !cbv) return TQ_ERR_NO_CONVERGENCE;
  AttendArgs a;
  a.q = q;
  a.q_dtype = q_dtype;
  a.packed_k = packed_k;
  a.norms_k = norms_k;
  a.packed_v = packed_v;
  a.norms_v = norms_v;
  a.new_kv = (const uint16_t*)new_kv;
  a.new_kv_bf16 = kv_dtype == TQ_BF16;
  a.ctx_lens = ctx_lens;
  a.d = d;
  a.batch = batch;
  a.n_q_heads = n_q_heads;
  a.gqa = gqa_ratio;
  a.n_kv_heads = n_q_heads / gqa_ratio;
  a.bits_k = bits_k;
  a.bits_v = bits_v;
  a.cap_tok = cap_tok;
  a.tau = sparse_v_thresh;
  a.counters = (int*)workspace;
  a.slots = (float*)((uint8_t*)workspace + attend_counter_bytes(batch, n_q_heads));
  a.dev_status = dev_status;
  a.skipped = sparse_v_skipped;
  a.head_skipped = head_skipped;
  a.out = out;
  a.out_dtype = out_dtype;
  a.partial_out = partial_out;
  return from_cuda(launch_attend(a, *cbk, *cbv, sign_mask(seed), n_ctas,
                                 (cudaStream_t)stream));
}

}  // namespace tq

extern "C" {

int tq_abi_version(void) { return TQ_ABI_VERSION; }

const char* tq_status_string(int status) {
  switch (status) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG";
    case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
    case TQ_ERR_NO_CONVERGENCE: return "TQ_ERR_NO_CONVERGENCE";
    default: return "unknown tq_status";
  }
}

int tq_build_codebook(int bits, int d, double* centroids, double* thresholds,
                      double* mse) {
  if (bits < 1 || bits > 8 || d < 1 || !centroids || !thresholds)
    return TQ_ERR_INVALID_ARG;
  const int st = solve_lloyd_max(bits, centroids, thresholds, mse);
  if (st != TQ_OK) return st;
  const double s = 1.0 / sqrt((double)d);
  for (int j = 0; j < (1 << bits); ++j) centroids[j] *= s;
  for (int j = 0; j < (1 << bits) - 1; ++j) thresholds[j] *= s;
  return TQ_OK;
}

int tq_encode(const void* kv, int dtype, int n_tok, int n_kv_heads, int d,
              int bits_k, int bits_v, uint64_t seed, uint8_t* packed_k,
              uint8_t* packed_v, uint16_t* norms_k, uint16_t* norms_v,
              int cap_tok, int tok_offset, int* dev_status, void* stream) {
  if (n_tok < 0 || n_kv_heads < 1 || cap_tok < 1 || tok_offset < 0)
    return TQ_ERR_INVALID_ARG;
  if ((long long)tok_offset + n_tok > cap_tok) return TQ_ERR_INVALID_ARG;
  if (n_kv_heads > kMaxGridYZ) return TQ_ERR_UNSUPPORTED;
  if (dtype != TQ_F16 && dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (!bits_ok(bits_k) || !bits_ok(bits_v)) return TQ_ERR_INVALID_ARG;
  const int hd = check_head_dim(d);
  if (hd != TQ_OK) return hd;
  if (!kv || !packed_k || !packed_v || !norms_k || !norms_v) return TQ_ERR_INVALID_ARG;
  if (!aligned16(kv) || !aligned16(packed_k) || !aligned16(packed_v))
    return TQ_ERR_INVALID_ARG;
  if (n_tok == 0) return TQ_OK;
  const Codebook* cbk = codebook_for(bits_k);
  const Codebook* cbv = codebook_for(bits_v);
  if (!cbk || !cbv) return TQ_ERR_NO_CONVERGENCE;
  EncodeArgs a;
  a.kv = (const uint16_t*)kv;
  a.d = d;
  a.is_bf16 = dtype == TQ_BF16;
  a.n_tok = n_tok;
  a.n_kv_heads = n_kv_heads;
  a.bits_k = bits_k;
  a.bits_v = bits_v;
  a.packed_k = packed_k;
  a.packed_v = packed_v;
  a.norms_k = norms_k;
  a.norms_v = norms_v;
  a.cap_tok = cap_tok;
  a.tok_offset = tok_offset;
  a.dev_status = dev_status;
  return from_cuda(launch_encode(a, *cbk, *cbv, sign_mask(seed), (cudaStream_t)stream));
}

int tq_dequant(const uint8_t* packed, const uint16_t* norms, int n_tok,
               int n_kv_heads, int d, int bits, uint64_t seed, int cap_tok,
               int domain, float* out, void* stream) {
  if (n_tok < 0 || n_kv_heads < 1 || cap_tok < 1 || n_tok > cap_tok)
    return TQ_ERR_INVALID_ARG;
  if (n_kv_heads > kMaxGridYZ) return TQ_ERR_UNSUPPORTED;
  if (bits < 2 || bits > 4 || (domain != 0 && domain != 1)) return TQ_ERR_INVALID_ARG;
  const int hd = check_head_dim(d);
  if (hd != TQ_OK) return hd;
  if (!packed || !norms || !out) return TQ_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(out)) return TQ_ERR_INVALID_ARG;
  if (n_tok == 0) return TQ_OK;
  const Codebook* cb = codebook_for(bits);
  if (!cb) return TQ_ERR_NO_CONVERGENCE;
  DequantArgs a;
  a.d = d;
  a.packed = packed;
  a.norms = norms;
  a.n_tok = n_tok;
  a.n_kv_heads = n_kv_heads;
  a.bits = bits;
  a.cap_tok = cap_tok;
  a.domain = domain;
  a.out = out;
  return from_cuda(launch_dequant(a, *cb, sign_mask(seed), (cudaStream_t)stream));
}

size_t tq_attend_workspace_size(int batch, int n_q_heads, int cap_tok, int d) {
  if (batch < 1 || n_q_heads < 1 || cap_tok < 1 || check_head_dim(d) != TQ_OK) return 0;
  return attend_workspace_bytes(batch, n_q_heads, d);
}

int tq_attend(const void* q, int q_dtype, const uint8_t* packed_k,
              const uint16_t* norms_k, const uint8_t* packed_v,
              const uint16_t* norms_v, const int32_t* ctx_lens, int batch,
              int n_q_heads, int gqa_ratio, int d, int bits_k, int bits_v,
              uint64_t seed, int cap_tok, float sparse_v_thresh, int n_ctas,
              void* workspace, size_t workspace_bytes, int* dev_status,
              unsigned long long* sparse_v_skipped, void* out, int out_dtype,
              void* stream) {
  return tq::attend_common(q, q_dtype, nullptr, TQ_F16, const_cast<uint8_t*>(packed_k),
                           const_cast<uint16_t*>(norms_k), const_cast<uint8_t*>(packed_v),
                           const_cast<uint16_t*>(norms_v), ctx_lens, batch, n_q_heads,
                           gqa_ratio, d, bits_k, bits_v, seed, cap_tok, sparse_v_thresh,
                           n_ctas, workspace, workspace_bytes, dev_status, sparse_v_skipped,
                           out, out_dtype, 0, stream);
}

int tq_attend_gate_counts(const void* q, int q_dtype, const uint8_t* packed_k,
                          const uint16_t* norms_k, const uint8_t* packed_v,
                          const uint16_t* norms_v, const int32_t* ctx_lens, int batch,
                          int n_q_heads, int gqa_ratio, int d, int bits_k, int bits_v,
                          uint64_t seed, int cap_tok, float sparse_v_thresh, int n_ctas,
                          void* workspace, size_t workspace_bytes, int* dev_status,
                          unsigned long long* sparse_v_skipped, unsigned int* head_skipped,
                          void* out, int out_dtype, void* stream) {
  if (!head_skipped) return TQ_ERR_INVALID_ARG;
  return tq::attend_common(q, q_dtype, nullptr, TQ_F16, const_cast<uint8_t*>(packed_k),
                           const_cast<uint16_t*>(norms_k), const_cast<uint8_t*>(packed_v),
                           const_cast<uint16_t*>(norms_v), ctx_lens, batch, n_q_heads,
                           gqa_ratio, d, bits_k, bits_v, seed, cap_tok, sparse_v_thresh,
                           n_ctas, workspace, workspace_bytes, dev_status, sparse_v_skipped,
                           out, out_dtype, 0, stream, head_skipped);
}

int tq_attend_append(const void* q, int q_dtype, const void* new_kv, int kv_dtype,
                     uint8_t* packed_k, uint16_t* norms_k, uint8_t* packed_v,
                     uint16_t* norms_v, const int32_t* ctx_lens, int batch,
                     int n_q_heads, int gqa_ratio, int d, int bits_k, int bits_v,
                     uint64_t seed, int cap_tok, float sparse_v_thresh, int n_ctas,
                     void* workspace, size_t workspace_bytes, int* dev_status,
                     unsigned long long* sparse_v_skipped, void* out, int out_dtype,
                     void* stream) {
  if (!new_kv) return TQ_ERR_INVALID_ARG;
  if (kv_dtype != TQ_F16 && kv_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (!aligned16(new_kv)) return TQ_ERR_INVALID_ARG;
  return tq::attend_common(q, q_dtype, new_kv, kv_dtype, packed_k, norms_k, packed_v, norms_v,
                           ctx_lens, batch, n_q_heads, gqa_ratio, d, bits_k, bits_v, seed,
                           cap_tok, sparse_v_thresh, n_ctas, workspace, workspace_bytes,
                           dev_status, sparse_v_skipped, out, out_dtype, 0, stream);
}

int tq_attend_partial(const void* q, int q_dtype, const uint8_t* packed_k,
                      const uint16_t* norms_k, const uint8_t* packed_v,
                      const uint16_t* norms_v, const int32_t* ctx_lens, int batch,
                      int n_q_heads, int gqa_ratio, int d, int bits_k, int bits_v,
                      uint64_t seed, int cap_tok, float sparse_v_thresh, int n_ctas,
                      void* workspace, size_t workspace_bytes, int* dev_status,
                      unsigned long long* sparse_v_skipped, float* partial, void* stream) {
  return tq::attend_common(q, q_dtype, nullptr, TQ_F16, const_cast<uint8_t*>(packed_k),
                           const_cast<uint16_t*>(norms_k), const_cast<uint8_t*>(packed_v),
                           const_cast<uint16_t*>(norms_v), ctx_lens, batch, n_q_heads,
                           gqa_ratio, d, bits_k, bits_v, seed, cap_tok, sparse_v_thresh,
                           n_ctas, workspace, workspace_bytes, dev_status, sparse_v_skipped,
                           partial, TQ_F32, 1, stream);
}

int tq_attend_combine(const float* partials, int n_parts, int batch, int n_q_heads, int d,
                      uint64_t seed, int* dev_status, void* out, int out_dtype,
                      void* stream) {
  if (n_parts < 1 || batch < 1 || n_q_heads < 1) return TQ_ERR_INVALID_ARG;
  if ((long long)batch * n_q_heads > (1LL << 30)) return TQ_ERR_UNSUPPORTED;
  if (out_dtype < TQ_F16 || out_dtype > TQ_F32) return TQ_ERR_INVALID_ARG;
  const int hd = check_head_dim(d);
  if (hd != TQ_OK) return hd;
  if (!partials || !out) return TQ_ERR_INVALID_ARG;
  if (((uintptr_t)partials & 7u) || !aligned16(out) || ((uintptr_t)dev_status & 3u))
    return TQ_ERR_INVALID_ARG;
  CombineArgs a;
  a.partials = partials;
  a.n_parts = n_parts;
  a.n_rec = batch * n_q_heads;
  a.d = d;
  a.dev_status = dev_status;
  a.out = out;
  a.out_dtype = out_dtype;
  return from_cuda(launch_combine(a, sign_mask(seed), (cudaStream_t)stream));
}

int tq_prefill_attend(const void* q, int q_dtype, const uint8_t* packed_k,
                      const uint16_t* norms_k, const uint8_t* packed_v,
                      const uint16_t* norms_v, const int32_t* ctx_lens, int batch,
                      int n_tok, int n_q_heads, int gqa_ratio, int d, int bits_k,
                      int bits_v, uint64_t seed, int cap_tok, int* dev_status, void* out,
                      int out_dtype, void* stream) {
  return tq_prefill_attend_split(q, q_dtype, packed_k, norms_k, packed_v, norms_v, ctx_lens,
                                 batch, n_tok, n_q_heads, gqa_ratio, d, bits_k, bits_v, seed,
                                 cap_tok, 1, nullptr, 0, dev_status, out, out_dtype, stream);
}

int tq_prefill_splits(int batch, int n_tok, int n_q_heads, int gqa_ratio, int max_ctx) {
  if (batch < 1 || n_tok < 1 || n_q_heads < 1 || gqa_ratio < 1 || n_q_heads % gqa_ratio ||
      gqa_ratio > kMaxGroup)
    return 1;
  // CTAs of one split (one per SM: 128 query rows each); pick the split
  // count that minimizes rounds of the SMs times the time of one CTA
  const long long rows_per_tile = 128 / gqa_ratio;
  // the longest tile's 128-position chunks; a split of fewer chunks than
  // splits would leave some empty
  const int nch = ((max_ctx > n_tok ? max_ctx : n_tok) + 127) / 128;
  const double chunks = (double)nch;
  const long long ctas = (long long)batch * (n_q_heads / gqa_ratio) *
                         ((n_tok + rows_per_tile - 1) / rows_per_tile);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0)
    sms = 148;
  int best = 1;
  double best_cost = (double)((ctas + sms - 1) / sms) * (chunks + 5.0);
  for (int sp = 2; sp <= kMaxPrefillSplits && sp <= nch; ++sp) {
    const double cost = (double)((ctas * sp + sms - 1) / sms) * (chunks / sp + 5.0);
    if (cost < best_cost - 1e-9) {
      best = sp;
      best_cost = cost;
    }
  }
  return best;
}

size_t tq_prefill_workspace_size(int batch, int n_tok, int n_q_heads, int d, int n_splits) {
  if (batch < 1 || n_tok < 1 || n_q_heads < 1 || n_splits <= 1 || check_head_dim(d) != TQ_OK)
    return 0;
  return (size_t)n_splits * batch * n_tok * n_q_heads * (d + 2) * sizeof(float);
}

int tq_prefill_attend_split(const void* q, int q_dtype, const uint8_t* packed_k,
                            const uint16_t* norms_k, const uint8_t* packed_v,
                            const uint16_t* norms_v, const int32_t* ctx_lens, int batch,
                            int n_tok, int n_q_heads, int gqa_ratio, int d, int bits_k,
                            int bits_v, uint64_t seed, int cap_tok, int n_splits,
                            void* workspace, size_t workspace_bytes, int* dev_status,
                            void* out, int out_dtype, void* stream) {
  if (n_splits < 1 || n_splits > kMaxPrefillSplits) return TQ_ERR_INVALID_ARG;
  if (n_splits > 1 &&
      (!workspace || ((uintptr_t)workspace & 15u) || n_tok < 1 ||
       workspace_bytes < tq_prefill_workspace_size(batch, n_tok, n_q_heads, d, n_splits)))
    return TQ_ERR_INVALID_ARG;
  if (n_splits > 1 && (long long)batch * n_tok * n_q_heads > (1LL << 30))
    return TQ_ERR_UNSUPPORTED;
  if (batch < 1 || n_tok < 1 || n_q_heads < 1 || gqa_ratio < 1 || cap_tok < 1)
    return TQ_ERR_INVALID_ARG;
  if (n_q_heads % gqa_ratio) return TQ_ERR_INVALID_ARG;
  if (gqa_ratio > kMaxGroup) return TQ_ERR_UNSUPPORTED;
  if (q_dtype < TQ_F16 || q_dtype > TQ_F32 || out_dtype < TQ_F16 || out_dtype > TQ_F32)
    return TQ_ERR_INVALID_ARG;
  if (!bits_ok(bits_k) || !bits_ok(bits_v)) return TQ_ERR_INVALID_ARG;
  const int hd = check_head_dim(d);
  if (hd != TQ_OK) return hd;
  if (d != 128) return TQ_ERR_UNSUPPORTED;       // prefill: d = 128
  if (cap_tok % 8) return TQ_ERR_UNSUPPORTED;
  if (!q || !packed_k || !norms_k || !packed_v || !norms_v || !ctx_lens || !out)
    return TQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(packed_k) || !aligned16(packed_v) ||
      !aligned16(norms_k) || !aligned16(norms_v) || ((uintptr_t)ctx_lens & 3u) ||
      ((uintptr_t)dev_status & 3u))
    return TQ_ERR_INVALID_ARG;
  const Codebook* cbk = codebook_for(bits_k);
  const Codebook* cbv = codebook_for(bits_v);
  if (!cbk || !cbv) return TQ_ERR_NO_CONVERGENCE;
  PrefillArgs a;
  a.q = q;
  a.q_dtype = q_dtype;
  a.packed_k = packed_k;
  a.norms_k = norms_k;
  a.packed_v = packed_v;
  a.norms_v = norms_v;
  a.ctx_lens = ctx_lens;
  a.batch = batch;
  a.n_tok = n_tok;
  a.n_q_heads = n_q_heads;
  a.gqa = gqa_ratio;
  a.n_kv_heads = n_q_heads / gqa_ratio;
  a.bits_k = bits_k;
  a.bits_v = bits_v;
  a.cap_tok = cap_tok;
  a.dev_status = dev_status;
  a.out = out;
  a.out_dtype = out_dtype;
  a.n_splits = n_splits;
  a.records = n_splits > 1 ? (float*)workspace : nullptr;
  return from_cuda(launch_prefill(a, *cbk, *cbv, sign_mask(seed), (cudaStream_t)stream));
}

int tq_qjl_encode(const void* k, int dtype, int n_tok, int n_kv_heads, int d, int bits_k,
                  uint64_t seed, const float* projection, const uint8_t* packed_k,
                  const uint16_t* norms_k, uint8_t* sketch, uint16_t* gamma, int cap_tok,
                  int tok_offset, int* dev_status, void* stream) {
  if (n_tok < 0 || n_kv_heads < 1 || cap_tok < 1 || tok_offset < 0)
    return TQ_ERR_INVALID_ARG;
  if ((long long)tok_offset + n_tok > cap_tok) return TQ_ERR_INVALID_ARG;
  if (n_kv_heads > kMaxGridYZ) return TQ_ERR_UNSUPPORTED;
  if (dtype != TQ_F16 && dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (!bits_ok(bits_k)) return TQ_ERR_INVALID_ARG;
  const int hd = check_head_dim(d);
  if (hd != TQ_OK) return hd;
  if (!k || !projection || !packed_k || !norms_k || !sketch || !gamma) return TQ_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(projection) || !aligned16(packed_k) ||
      ((uintptr_t)norms_k & 1u) || ((uintptr_t)gamma & 1u) || ((uintptr_t)dev_status & 3u))
    return TQ_ERR_INVALID_ARG;
  if (n_tok == 0) return TQ_OK;
  const Codebook* cb = codebook_for(bits_k);
  if (!cb) return TQ_ERR_NO_CONVERGENCE;
  QjlEncodeArgs a;
  a.k = (const uint16_t*)k;
  a.is_bf16 = dtype == TQ_BF16;
  a.d = d;
  a.n_tok = n_tok;
  a.n_kv_heads = n_kv_heads;
  a.bits_k = bits_k;
  a.packed_k = packed_k;
  a.norms_k = norms_k;
  a.S = projection;
  a.sketch = sketch;
  a.gamma = gamma;
  a.cap_tok = cap_tok;
  a.tok_offset = tok_offset;
  a.dev_status = dev_status;
  return from_cuda(launch_qjl_encode(a, *cb, sign_mask(seed), (cudaStream_t)stream));
}

int tq_qjl_scores(const void* q, int q_dtype, const uint8_t* packed_k, const uint16_t* norms_k,
                  const uint8_t* sketch, const uint16_t* gamma, const float* projection,
                  const int32_t* ctx_lens, int batch, int n_q_heads, int gqa_ratio, int d,
                  int bits_k, uint64_t seed, int cap_tok, int with_sketch, int* dev_status,
                  float* scores, void* stream) {
  if (batch < 1 || n_q_heads < 1 || gqa_ratio < 1 || cap_tok < 1) return TQ_ERR_INVALID_ARG;
  if (n_q_heads % gqa_ratio) return TQ_ERR_INVALID_ARG;
  if (gqa_ratio > kMaxGroup) return TQ_ERR_UNSUPPORTED;
  if (batch > kMaxGridYZ || n_q_heads / gqa_ratio > kMaxGridYZ) return TQ_ERR_UNSUPPORTED;
  if (q_dtype < TQ_F16 || q_dtype > TQ_F32) return TQ_ERR_INVALID_ARG;
  if (!bits_ok(bits_k) || (with_sketch != 0 && with_sketch != 1)) return TQ_ERR_INVALID_ARG;
  const int hd = check_head_dim(d);
  if (hd != TQ_OK) return hd;
  if (!q || !packed_k || !norms_k || !ctx_lens || !scores) return TQ_ERR_INVALID_ARG;
  if (with_sketch && (!sketch || !gamma || !projection)) return TQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(packed_k) || !aligned16(projection) ||
      ((uintptr_t)sketch & 7u) || ((uintptr_t)norms_k & 1u) || ((uintptr_t)gamma & 1u) ||
      ((uintptr_t)ctx_lens & 3u) || ((uintptr_t)scores & 3u) || ((uintptr_t)dev_status & 3u))
    return TQ_ERR_INVALID_ARG;
  const Codebook* cb = codebook_for(bits_k);
  if (!cb) return TQ_ERR_NO_CONVERGENCE;
  QjlScoresArgs a;
  a.q = q;
  a.q_dtype = q_dtype;
  a.packed_k = packed_k;
  a.norms_k = norms_k;
  a.sketch = sketch;
  a.gamma = gamma;
  a.S = projection;
  a.ctx_lens = ctx_lens;
  a.d = d;
  a.batch = batch;
  a.n_q_heads = n_q_heads;
  a.gqa = gqa_ratio;
  a.n_kv_heads = n_q_heads / gqa_ratio;
  a.bits_k = bits_k;
  a.cap_tok = cap_tok;
  a.with_sketch = with_sketch;
  a.dev_status = dev_status;
  a.out = scores;
  return from_cuda(launch_qjl_scores(a, *cb, sign_mask(seed), (cudaStream_t)stream));
}

}  // extern "C"
