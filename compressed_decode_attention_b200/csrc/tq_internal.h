// Internal definitions shared by the host layer (api.cpp) and the kernels.
// Not part of the public ABI (include/tq.h is).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime.h>

namespace tq {

constexpr int kMaxHeadDim = 256;       // d in {64, 128, 256}
constexpr int kMaxLevels = 16;         // 2^4: widest code on the hot path
constexpr int kGateBlock = 64;         // sparse-V block (TQ_SPARSE_V_BLOCK)
constexpr int kMaxGroup = 8;           // largest GQA group handled per CTA

// Codebook in N(0,1) units, as float for the kernels.
struct Codebook {
  float centroid[kMaxLevels];          // 2^bits ascending levels
  float threshold[kMaxLevels];         // 2^bits - 1 ascending thresholds
  int bits;
};

// Sign vector D as a bit mask: bit i of word i/32 set <=> D_i = -1.
struct SignMask {
  uint32_t w[kMaxHeadDim / 32];        // the first d bits are used
};

// ---------------------------------------------------------------- host side
// Lloyd-Max solver (codebook.cpp). Returns 0 on success, else a tq_status.
int solve_lloyd_max(int bits, double* centroids, double* thresholds,
                    double* mse);
// Cached float codebook for bits in 1..4 (computed once, immutable after).
const Codebook* codebook_for(int bits);
SignMask sign_mask(uint64_t seed);

// ---------------------------------------------------------------- launchers
struct EncodeArgs {
  const uint16_t* kv;        // [2][n_tok][n_kv_heads][d]
  int d;
  int is_bf16;
  int n_tok, n_kv_heads;
  int bits_k, bits_v;
  uint8_t* packed_k;
  uint8_t* packed_v;
  uint16_t* norms_k;
  uint16_t* norms_v;
  int cap_tok, tok_offset;
  int* dev_status;
};
cudaError_t launch_encode(const EncodeArgs& a, const Codebook& cbk,
                          const Codebook& cbv, const SignMask& sm,
                          cudaStream_t stream);
// Tensor-core encode (encode_tc.cu): d = 128 and enough tokens to fill tiles.
bool encode_tc_applies(const EncodeArgs& a);
cudaError_t launch_encode_tc(const EncodeArgs& a, const Codebook& cbk, const Codebook& cbv,
                             const SignMask& sm, int sms, cudaStream_t stream);

struct DequantArgs {
  int d;
  const uint8_t* packed;
  const uint16_t* norms;
  int n_tok, n_kv_heads, bits, cap_tok, domain;
  float* out;
};
cudaError_t launch_dequant(const DequantArgs& a, const Codebook& cb,
                           const SignMask& sm, cudaStream_t stream);

struct AttendArgs {
  const void* q;
  int q_dtype;
  // The cache; written only by the decode-step append (new_kv != nullptr).
  uint8_t* packed_k;
  uint16_t* norms_k;
  uint8_t* packed_v;
  uint16_t* norms_v;
  // Decode-step append: [2][batch][n_kv_heads][d] fp16/bf16 new K/V (one
  // token per sequence), encoded into row ctx_lens[b] - 1; nullptr = none.
  const uint16_t* new_kv;
  int new_kv_bf16;
  const int32_t* ctx_lens;
  int d;
  int batch, n_q_heads, gqa, n_kv_heads;
  int bits_k, bits_v;
  int cap_tok;
  float tau;
  int* counters;             // [batch * n_kv_heads], zero between calls
  float* slots;              // partial (acc[gqa][d], m/l[gqa][2]) per slot
  int* dev_status;
  unsigned long long* skipped;
  unsigned int* head_skipped;  // [batch][n_q_heads] gated positions per head, or nullptr
  void* out;
  int out_dtype;
  // Context-parallel slice: out is float [batch][n_q_heads][d + 2] of
  // log-sum-exp records (acc in the unnormalized Hadamard domain, then the
  // base-2 maximum and the sum) instead of the attention output.
  int partial_out;
};
cudaError_t launch_attend(const AttendArgs& a, const Codebook& cbk,
                          const Codebook& cbv, const SignMask& sm, int n_ctas,
                          cudaStream_t stream);
// Per head dimension (attend_d64.cu, attend_d128.cu, attend_d256.cu).
template <int D>
cudaError_t launch_attend_d(const AttendArgs& a, const Codebook& cbk, const Codebook& cbv,
                            const SignMask& sm, int n_ctas, cudaStream_t stream);

struct PrefillArgs {
  const void* q;             // [batch][n_tok][n_q_heads][d]
  int q_dtype;
  const uint8_t* packed_k;
  const uint16_t* norms_k;
  const uint8_t* packed_v;
  const uint16_t* norms_v;
  const int32_t* ctx_lens;
  int batch, n_tok, n_q_heads, gqa, n_kv_heads;
  int bits_k, bits_v;
  int cap_tok;
  int* dev_status;
  void* out;                 // [batch][n_tok][n_q_heads][d]
  int out_dtype;
  // n_splits > 1: every tile's context is split n_splits ways; the splits
  // write log-sum-exp records [n_splits][batch*n_tok*n_q_heads][d + 2] and
  // a combine launch merges them into out
  int n_splits;
  float* records;
};
constexpr int kMaxPrefillSplits = 8;
cudaError_t launch_prefill(const PrefillArgs& a, const Codebook& cbk, const Codebook& cbv,
                           const SignMask& sm, cudaStream_t stream);

struct CombineArgs {
  const float* partials;     // [n_parts][n_rec][d + 2]
  int n_parts;
  int n_rec;                 // batch * n_q_heads
  int d;
  int* dev_status;
  void* out;                 // [n_rec][d] of out_dtype
  int out_dtype;
};
cudaError_t launch_combine(const CombineArgs& a, const SignMask& sm, cudaStream_t stream);

// Stage-2 residual sketch of keys (one kv head block per grid row).
struct QjlEncodeArgs {
  const uint16_t* k;         // [n_tok][n_kv_heads][d] fp16/bf16 keys
  int is_bf16;
  int d, n_tok, n_kv_heads, bits_k;
  const uint8_t* packed_k;   // stage-1 rows [n_kv_heads][cap_tok][d*bits_k/8] (read)
  const uint16_t* norms_k;   // [n_kv_heads][cap_tok]
  const float* S;            // [d][d] projection, row i = projection i
  uint8_t* sketch;           // [n_kv_heads][cap_tok][d/8]
  uint16_t* gamma;           // [n_kv_heads][cap_tok] fp16 residual norms
  int cap_tok, tok_offset;
  int* dev_status;
};
cudaError_t launch_qjl_encode(const QjlEncodeArgs& a, const Codebook& cb, const SignMask& sm,
                              cudaStream_t stream);

struct QjlScoresArgs {
  const void* q;             // [batch][n_q_heads][d]
  int q_dtype;
  const uint8_t* packed_k;   // [batch][n_kv_heads][cap_tok][d*bits_k/8]
  const uint16_t* norms_k;
  const uint8_t* sketch;     // [batch][n_kv_heads][cap_tok][d/8]
  const uint16_t* gamma;
  const float* S;            // [d][d]
  const int32_t* ctx_lens;
  int d, batch, n_q_heads, gqa, n_kv_heads, bits_k, cap_tok;
  int with_sketch;
  int* dev_status;
  float* out;                // [batch][n_q_heads][cap_tok]
};
cudaError_t launch_qjl_scores(const QjlScoresArgs& a, const Codebook& cb, const SignMask& sm,
                              cudaStream_t stream);

// Workspace of tq_attend: a counter region (zero on first use; every call
// leaves it zero) followed by partial-result slots. Sized for up to
// kMaxCtas CTAs, independent of the device.
constexpr int kMaxCtas = 1024;
// A slot holds, per query head, d accumulators then (max, sum).
inline size_t attend_counter_bytes(int batch, int n_q_heads) {
  return ((size_t)batch * n_q_heads * sizeof(int) + 255) & ~(size_t)255;
}
inline size_t attend_workspace_bytes(int batch, int n_q_heads, int d) {
  const size_t slots = (size_t)kMaxCtas * kMaxGroup + (size_t)batch * n_q_heads;
  return attend_counter_bytes(batch, n_q_heads) + slots * (size_t)(d + 2) * sizeof(float);
}

}  // namespace tq
