/*
 * tq.h — C ABI of a compressed KV-cache library for NVIDIA B200 (sm_100a).
 *
 * The library does two things on the GPU:
 *   1. tq_encode   — compress K/V head vectors: FP16 norm, seeded randomized
 *                    Hadamard rotation, Lloyd-Max scalar codebook, bit-packing.
 *   2. tq_attend   — decode attention that reads only the packed cache.
 * plus tq_dequant (verification) and tq_build_codebook (host-side solver).
 *
 * Sources (cited below by the key in brackets, then the section):
 *   [TQAI]   "We Built a Python Library That Cuts LLM Memory Usage by 80%"
 *            (dev.to, tqai library post)
 *   [ADAPTQ] "AdapTQ — Adaptive Streaming Vector Quantization KV Cache for
 *            LLMs" (PyPI project page, adaptq 0.2.3)
 *   [TQPLUS] "TurboQuant+: Compresión de Caché KV 6.4x para LLMs" (aibit.im)
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers unless marked "host".
 *   - The caller owns every buffer. No entry point allocates device memory;
 *     scratch space for tq_attend is passed in by the caller.
 *   - GPU entry points are asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL means the legacy default stream). They validate arguments
 *     on the host, enqueue kernels and return without synchronizing. A
 *     TQ_ERR_CUDA return reports a launch failure (cudaGetLastError);
 *     execution errors surface at the caller's next synchronization.
 *   - Entry points hold no global state: codebooks and the sign vector travel
 *     to the kernels as launch parameters, so calls are thread-safe.
 *   - Kernels never trap and never spin. Device-side conditions set bits in
 *     the optional *dev_status word (atomicOr; the caller zeroes it).
 *
 * Frozen format definitions (the pages leave these open; these readings are
 * the library's own and the test oracle implements the same definitions):
 *   - Codebook: Lloyd-Max quantizer for N(0,1) with 2^b levels, symmetric,
 *     ascending; thresholds are the midpoints between adjacent centroids.
 *     The N(0,1/d) codebook of [TQAI §The Paper] is that codebook / sqrt(d).
 *     Kernels compare zeta = z/||x|| against the N(0,1) thresholds, where
 *     z = H·(D⊙x) with the unnormalized Hadamard matrix, so zeta = sqrt(d)·y.
 *   - Index: idx_i = #{ j : zeta_i >= t_j } (a value on a threshold goes to
 *     the upper cell).
 *   - Sign vector D: SplitMix64 (Steele, Lea & Flood 2014) with state = seed;
 *     D_i = -1 iff bit 63 of the i-th output (i = 0..d-1) is set. The same D
 *     serves K, V, all heads and the query; pass one seed per layer.
 *   - Hadamard: Sylvester order, H[i][j] = (-1)^popcount(i & j).
 *   - Packing: LSB-first contiguous. Row bit (i·b + k) is bit k of idx_i;
 *     row byte j holds row bits 8j..8j+7. One row of d·b/8 bytes per
 *     (sequence, kv head, token).
 *   - Norm: ||x||_2 of the fp16/bf16 input promoted to float, stored as IEEE
 *     fp16 with round-to-nearest-even, saturated to 65504 (TQ_DEV_NORM_SATURATED).
 *     The unit vector is formed with the unrounded norm.
 *   - Sparse-V gate [TQPLUS §2 Sparse V]: with tau = sparse_v_thresh > 0, the
 *     V row at position t is left out of query head h's accumulation iff
 *     exp(s_t - M_blk(t)) < tau, where M_blk(t) is the maximum score of head h
 *     over the aligned block of TQ_SPARSE_V_BLOCK positions containing t
 *     (blocks start at position 0). Gated positions still count in the
 *     softmax denominator. tau <= 0 disables the gate.
 *
 * Cache layout (attend/dequant):
 *   packed_k : uint8 [batch][n_kv_heads][cap_tok][d*bits_k/8]
 *   packed_v : uint8 [batch][n_kv_heads][cap_tok][d*bits_v/8]
 *   norms_k, norms_v : fp16 bits (uint16) [batch][n_kv_heads][cap_tok]
 * tq_encode writes one sequence (batch index 0 of that layout, i.e. pass the
 * base pointers of the sequence you are filling).
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TQ_ABI_VERSION 8

/* Tokens per sparse-V block; split boundaries are multiples of this. */
#define TQ_SPARSE_V_BLOCK 64

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,    /* a null pointer, a size out of range, ... */
  TQ_ERR_UNSUPPORTED = 2,    /* valid in principle, not built (e.g. d != 128) */
  TQ_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed */
  TQ_ERR_NO_CONVERGENCE = 4  /* the Lloyd-Max iteration did not converge */
} tq_status;

typedef enum { TQ_F16 = 0, TQ_BF16 = 1, TQ_F32 = 2 } tq_dtype;

/* Bits of *dev_status (device int, zeroed by the caller, set with atomicOr). */
#define TQ_DEV_CTX_CLAMPED    1  /* some ctx_lens[b] > cap_tok; clamped     */
#define TQ_DEV_NORM_SATURATED 2  /* some norm > 65504; stored as 65504      */
#define TQ_DEV_CTX_EMPTY      4  /* some ctx_lens[b] <= 0; output set to 0  */
#define TQ_DEV_WAIT_TIMEOUT   8  /* a wait for staged cache data gave up    */
#define TQ_DEV_DEBUG_CHECK   16  /* bounds-checked build (TQ_DEBUG) only: an
                                    index check failed; the access was skipped */
                                 /* after ~1 s; the output is not valid     */

/* Library ABI version (TQ_ABI_VERSION of the build). */
int tq_abi_version(void);

/* Static, human-readable name of a status code. */
const char* tq_status_string(int status);

/*
 * tq_build_codebook — host-side Lloyd-Max solver for the post-rotation
 * coordinate distribution N(0, 1/d) [TQAI §The Paper: after the rotation a
 * coordinate is modelled as Gaussian with variance 1/d, so the optimal
 * scalar quantizer is fixed in advance and needs no data; ADAPTQ §How it
 * works, item 2].
 *
 *   bits        1..8; the codebook has N = 2^bits levels.
 *   d           head dimension >= 1 (d = 1 gives the N(0,1) codebook).
 *   centroids   host, N doubles, ascending, symmetric about 0.
 *   thresholds  host, N-1 doubles, t_j = (c_{j-1} + c_j)/2, ascending.
 *   mse         host, nullable: expected squared error of a rotated unit
 *               vector, i.e. the per-coordinate MSE in N(0,1) units
 *               (0.1175 / 0.03454 / 0.009497 at 2 / 3 / 4 bits).
 * Pure host computation: needs no GPU. Returns TQ_ERR_INVALID_ARG on bad
 * arguments, TQ_ERR_NO_CONVERGENCE if the fixed point is not reached.
 */
int tq_build_codebook(int bits, int d, double* centroids, double* thresholds,
                      double* mse);

/*
 * tq_encode — compress n_tok tokens of one sequence into a packed cache
 * [TQAI §The Paper (rotate, quantize each coordinate, store the norm in
 * FP16); ADAPTQ §How it works, items 1-2 (y = (1/sqrt d)·H·D·x via FWHT,
 * Max-Lloyd codebook); TQAI §Compression numbers (K4/V2, K3/V2, K4/V3) and
 * §What's Next (bit-packing)].
 *
 *   kv          [2][n_tok][n_kv_heads][d] of `dtype` (TQ_F16 or TQ_BF16):
 *               the K block followed by the V block, token-major as a
 *               projection produces them. 16-byte aligned.
 *   n_tok       >= 0 tokens to encode (0 is a no-op).
 *   n_kv_heads  >= 1.
 *   d           head dimension: 64, 128 or 256 (else TQ_ERR_INVALID_ARG).
 *   bits_k, bits_v  2..4 bits per coordinate for K and for V.
 *   seed        sign-vector seed (see "Sign vector D" above).
 *   packed_k    [n_kv_heads][cap_tok][d*bits_k/8] bytes, 16-byte aligned.
 *   packed_v    [n_kv_heads][cap_tok][d*bits_v/8] bytes, 16-byte aligned.
 *   norms_k, norms_v  [n_kv_heads][cap_tok] fp16 bits.
 *   cap_tok     token capacity of the cache rows (>= 1).
 *   tok_offset  first row written; rows tok_offset .. tok_offset+n_tok-1.
 *               tok_offset + n_tok <= cap_tok, else TQ_ERR_INVALID_ARG.
 *   dev_status  device int, nullable; TQ_DEV_NORM_SATURATED may be set.
 *   stream      cudaStream_t.
 * Rows outside the written range are untouched.
 */
int tq_encode(const void* kv, int dtype, int n_tok, int n_kv_heads, int d,
              int bits_k, int bits_v, uint64_t seed,
              uint8_t* packed_k, uint8_t* packed_v,
              uint16_t* norms_k, uint16_t* norms_v,
              int cap_tok, int tok_offset, int* dev_status, void* stream);

/*
 * tq_dequant — reconstruct vectors from one packed cache (K or V) for
 * verification; not used by tq_attend.
 *
 *   packed      [n_kv_heads][cap_tok][d*bits/8] bytes.
 *   norms       [n_kv_heads][cap_tok] fp16 bits.
 *   n_tok       rows 0..n_tok-1 of each head are reconstructed (<= cap_tok).
 *   domain      0: original space, x_hat = fp16norm · D⊙(H·c[idx]) / d;
 *               1: rotated unit-vector coordinates c[idx] / sqrt(d)
 *               (the N(0,1/d) codebook values, norm not applied).
 *   out         float [n_kv_heads][n_tok][d], 16-byte aligned.
 * packed must be 16-byte aligned.
 */
int tq_dequant(const uint8_t* packed, const uint16_t* norms, int n_tok,
               int n_kv_heads, int d, int bits, uint64_t seed, int cap_tok,
               int domain, float* out, void* stream);

/*
 * tq_attend_workspace_size — bytes of device scratch tq_attend needs for
 * this batch and head count: a counter region of
 * round_up(4·batch·n_q_heads, 256) bytes, then per-split partial results
 * (running max, sum and d accumulators in fp32 per query head) for up to 1024
 * CTAs. Returns 0 for invalid arguments.
 */
size_t tq_attend_workspace_size(int batch, int n_q_heads, int cap_tok, int d);

/*
 * tq_attend — single-query decode attention over the packed cache
 * [ADAPTQ §How it works, item 3: the query is rotated a single time and the
 * scores are formed from the packed indices, never materializing the
 * dequantized cache; TQAI §What's Next: fused decode over compressed data;
 * TQAI §Test Suite: the attention being approximated is
 * softmax(Q·K^T/sqrt d)·V; TQPLUS §2 Sparse V].
 *
 * For batch b and query head h (kv head g = h / gqa_ratio, i.e. consecutive
 * query heads share a kv head) with L = min(ctx_lens[b], cap_tok):
 *   q~   = H·(D⊙q) / sqrt(d)                       (rotated once)
 *   s_t  = (1/sqrt d) · nK_t · sum_i q~_i · cK[idxK_t,i] / sqrt(d),  t < L
 *   w_t  = exp(s_t - max s),  l = sum_t w_t
 *   acc  = sum_{t not gated} w_t · nV_t · cV[idxV_t] / sqrt(d)
 *   out  = D⊙(H·(acc / l)) / sqrt(d)               (inverse-rotated once)
 * where c are the N(0,1) codebooks and nK, nV the stored fp16 norms.
 *
 *   q           [batch][n_q_heads][d] of q_dtype (TQ_F16 | TQ_BF16 | TQ_F32),
 *               16-byte aligned.
 *   packed_*, norms_*  the cache layout above with a leading batch dim, all
 *               four 16-byte aligned; cap_tok must be a multiple of 8
 *               (TQ_ERR_UNSUPPORTED otherwise).
 *   ctx_lens    int32 [batch] on the device. Values > cap_tok are clamped
 *               (TQ_DEV_CTX_CLAMPED); values <= 0 give out = 0
 *               (TQ_DEV_CTX_EMPTY).
 *   batch >= 1; n_q_heads >= 1; gqa_ratio in 1..8 divides n_q_heads.
 *   d, bits_k, bits_v, seed   as used by tq_encode for this cache.
 *   sparse_v_thresh  tau of the sparse-V gate; <= 0 disables it.
 *   n_ctas      0: one CTA per SM (the intended setting); 1..1024 forces the
 *               number of CTAs the 64-position blocks are balanced over.
 *   workspace, workspace_bytes  >= tq_attend_workspace_size(...) bytes,
 *               16-byte aligned. Its counter region (the first
 *               round_up(4·batch·n_q_heads, 256) bytes) must be zero before
 *               the first call that uses it (e.g. cudaMemset once); every call
 *               leaves it zero again when it completes on the stream. The
 *               rest is scratch. One workspace per concurrently running call.
 *   dev_status  device int, nullable. TQ_DEV_WAIT_TIMEOUT reports a copy of
 *               cache data into shared memory that did not complete within
 *               about a second (the kernel then gives up instead of hanging).
 *   sparse_v_skipped  device uint64, nullable: atomically incremented by the
 *               number of (b, h, t) positions the gate left out.
 *   out         [batch][n_q_heads][d] of out_dtype (TQ_F16 | TQ_BF16 | TQ_F32),
 *               16-byte aligned.
 */
int tq_attend(const void* q, int q_dtype,
              const uint8_t* packed_k, const uint16_t* norms_k,
              const uint8_t* packed_v, const uint16_t* norms_v,
              const int32_t* ctx_lens, int batch, int n_q_heads,
              int gqa_ratio, int d, int bits_k, int bits_v, uint64_t seed,
              int cap_tok, float sparse_v_thresh, int n_ctas,
              void* workspace, size_t workspace_bytes, int* dev_status,
              unsigned long long* sparse_v_skipped,
              void* out, int out_dtype, void* stream);

/*
 * tq_attend_gate_counts — tq_attend that also reports, for every (sequence,
 * query head), how many positions the sparse-V gate left out of that head's
 * V accumulation [TQPLUS §2 Sparse V; the gate rule is frozen above]. Meant
 * for verifying the gate head by head; the attention itself is tq_attend's.
 *
 *   head_skipped  uint32 [batch][n_q_heads] on the device, 4-byte aligned,
 *               not NULL (TQ_ERR_INVALID_ARG): entry (b, h) is atomically
 *               incremented by the number of positions t < L_b gated for
 *               head h (the caller zeroes it). Nothing is added with the
 *               gate off (sparse_v_thresh <= 0).
 * All other arguments, results and errors are tq_attend's.
 */
int tq_attend_gate_counts(const void* q, int q_dtype,
                          const uint8_t* packed_k, const uint16_t* norms_k,
                          const uint8_t* packed_v, const uint16_t* norms_v,
                          const int32_t* ctx_lens, int batch, int n_q_heads,
                          int gqa_ratio, int d, int bits_k, int bits_v, uint64_t seed,
                          int cap_tok, float sparse_v_thresh, int n_ctas,
                          void* workspace, size_t workspace_bytes, int* dev_status,
                          unsigned long long* sparse_v_skipped, unsigned int* head_skipped,
                          void* out, int out_dtype, void* stream);

/*
 * tq_attend_append — one decode step in one launch: append the new token of
 * every sequence to the compressed cache, then attend over the cache
 * including it. The pages' decode loop updates the cache with the new
 * key/value pair before attention runs ("We Built a Python Library That Cuts
 * LLM Memory Usage by 80%", §The Paper: cache.update() ahead of the
 * attention call); this entry point does both steps in one kernel.
 *
 * Equivalent, bit for bit in the cache and within the attention tolerance in
 * out, to: for every b with L_b = min(ctx_lens[b], cap_tok) >= 1,
 *   tq_encode(new_kv[:, b], n_tok = 1, tok_offset = L_b - 1) on sequence b's
 *   cache, followed by tq_attend(...) with the same arguments.
 *
 *   new_kv      [2][batch][n_kv_heads][d] of kv_dtype (TQ_F16 | TQ_BF16),
 *               16-byte aligned: the new key (index 0) and value (index 1)
 *               of each sequence. ctx_lens counts the new token.
 *   packed_*, norms_*  the cache (written: row L_b - 1 of every kv head of
 *               every sequence with L_b >= 1). Sequences with ctx_lens[b] <= 0
 *               append nothing (out = 0, TQ_DEV_CTX_EMPTY); ctx_lens[b] >
 *               cap_tok writes row cap_tok - 1 (TQ_DEV_CTX_CLAMPED).
 *   TQ_DEV_NORM_SATURATED is set as in tq_encode.
 * All other arguments, the workspace contract and the errors are those of
 * tq_attend; a null new_kv or another kv_dtype is TQ_ERR_INVALID_ARG.
 */
int tq_attend_append(const void* q, int q_dtype, const void* new_kv, int kv_dtype,
                     uint8_t* packed_k, uint16_t* norms_k,
                     uint8_t* packed_v, uint16_t* norms_v,
                     const int32_t* ctx_lens, int batch, int n_q_heads,
                     int gqa_ratio, int d, int bits_k, int bits_v, uint64_t seed,
                     int cap_tok, float sparse_v_thresh, int n_ctas,
                     void* workspace, size_t workspace_bytes, int* dev_status,
                     unsigned long long* sparse_v_skipped,
                     void* out, int out_dtype, void* stream);

/*
 * tq_prefill_attend — causal attention of a chunk of n_tok new query tokens
 * per sequence over the compressed cache, the prefill counterpart of
 * tq_attend (TurboQuant+ §3 reports prefill with the compressed cache; the
 * scores and weighted sum follow AdapTQ §How it works, item 3). The chunk's
 * K/V rows must already be in the cache (tq_encode at tok_offset
 * ctx_lens[b] - n_tok). Runs on tensor cores: each CTA dequantizes a cache
 * chunk once into shared memory for up to 128 query rows.
 *
 *   q           [batch][n_tok][n_q_heads][d] of q_dtype, 16-byte aligned.
 *               Token i of sequence b sits at position
 *               p = ctx_lens[b] - n_tok + i and attends to positions 0..p.
 *   out         [batch][n_tok][n_q_heads][d] of out_dtype, 16-byte aligned.
 *   packed_*, norms_*, ctx_lens, batch, n_q_heads, gqa_ratio, bits_k,
 *               bits_v, seed, cap_tok, dev_status   as for tq_attend.
 *               Tokens with p < 0 (ctx_lens[b] < n_tok) get out = 0 and set
 *               TQ_DEV_CTX_EMPTY; ctx_lens[b] > cap_tok is clamped
 *               (TQ_DEV_CTX_CLAMPED).
 *   d           128 (TQ_ERR_UNSUPPORTED for 64 and 256).
 * No sparse-V gate and no workspace. Errors as for tq_attend.
 */
int tq_prefill_attend(const void* q, int q_dtype,
                      const uint8_t* packed_k, const uint16_t* norms_k,
                      const uint8_t* packed_v, const uint16_t* norms_v,
                      const int32_t* ctx_lens, int batch, int n_tok, int n_q_heads,
                      int gqa_ratio, int d, int bits_k, int bits_v, uint64_t seed,
                      int cap_tok, int* dev_status, void* out, int out_dtype,
                      void* stream);

/*
 * tq_prefill_attend_split — tq_prefill_attend with every query tile's
 * context split n_splits ways. Each split attends over its share of the
 * tile's 64-position chunks and leaves log-sum-exp records (the layout of
 * tq_attend_partial, one per (sequence, token, query head)) in the
 * workspace; a merge launch (tq_attend_combine's kernel) then writes out.
 * The result equals tq_prefill_attend's within the attention tolerance.
 * Splitting keeps all SMs busy when the tiles do not fill whole waves (one
 * CTA of 128 query rows per SM): 256 tiles on 148 SMs take two waves, four
 * splits of them seven quarter-waves.
 *   n_splits    1 .. 8; 1 is tq_prefill_attend (no workspace needed).
 *   workspace, workspace_bytes  >= tq_prefill_workspace_size(batch, n_tok,
 *               n_q_heads, d, n_splits) bytes, 16-byte aligned, for
 *               n_splits > 1; scratch (no state between calls).
 *   batch · n_tok · n_q_heads <= 2^30 when n_splits > 1 (TQ_ERR_UNSUPPORTED).
 * All other arguments and errors as for tq_prefill_attend.
 */
int tq_prefill_attend_split(const void* q, int q_dtype,
                            const uint8_t* packed_k, const uint16_t* norms_k,
                            const uint8_t* packed_v, const uint16_t* norms_v,
                            const int32_t* ctx_lens, int batch, int n_tok, int n_q_heads,
                            int gqa_ratio, int d, int bits_k, int bits_v, uint64_t seed,
                            int cap_tok, int n_splits, void* workspace,
                            size_t workspace_bytes, int* dev_status, void* out,
                            int out_dtype, void* stream);

/* Workspace bytes of tq_prefill_attend_split: n_splits · batch · n_tok ·
 * n_q_heads · (d + 2) floats; 0 for n_splits <= 1 or invalid arguments. */
size_t tq_prefill_workspace_size(int batch, int n_tok, int n_q_heads, int d, int n_splits);

/* A split count for tq_prefill_attend_split on the current device, for
 * sequences of at most max_ctx positions (n_tok if smaller): the n in
 * 1..min(8, chunks) that minimizes ceil(tiles·n / SMs) · (chunks / n + 5),
 * i.e. rounds of the SMs times the time of one CTA, which handles 1/n of
 * the longest tile's 128-position chunks after a fixed cost of about 5
 * chunks (set-up, pipeline fill and drain). Host only; 1 on bad input. */
int tq_prefill_splits(int batch, int n_tok, int n_q_heads, int gqa_ratio, int max_ctx);

/*
 * Context parallelism: the positions of every sequence are split over the
 * devices of a group, each device attends over its own slice and the
 * per-slice results are merged. The source pages run on one device; this
 * split is the library's extension, and it is exact (the log-sum-exp
 * identity), so the merged output equals tq_attend over the whole context
 * within the attention tolerance.
 *
 * Record layout (one per (sequence, query head), float32, d + 2 values):
 *   acc[0..d-1]  sum over the slice's ungated positions t of
 *                2^(s_t·log2(e) - m2) · nV_t · cV[idxV_t], cV the N(0,1)
 *                codebook: the value sum in the unnormalized Hadamard
 *                domain z = H·(D⊙v) of the encoder, not yet rotated back.
 *   acc[d]       m2 = log2(e) · max_t s_t (base-2 maximum score).
 *   acc[d + 1]   l = sum over ALL the slice's positions of 2^(s_t·log2(e) - m2).
 * A slice with no position gives acc = 0, m2 = -inf, l = 0.
 * s_t, nV_t, idxV_t and the gate are those of tq_attend.
 *
 * tq_attend_partial — tq_attend over one slice, writing records.
 *   The cache arguments describe the slice as a cache of its own: row 0 of
 *   each (sequence, kv head) is the slice's first position, ctx_lens[b] is
 *   the number of positions sequence b has in the slice (<= 0: an empty
 *   record and TQ_DEV_CTX_EMPTY, which is normal for a short sequence).
 *   For the sparse-V gate to act as in one pass over the whole context, a
 *   slice must start at a multiple of TQ_SPARSE_V_BLOCK positions (its
 *   blocks are aligned to its own row 0).
 *   partial     float [batch][n_q_heads][d + 2] records, 8-byte aligned (so
 *               row p of a gathered [n_parts][...] buffer always qualifies).
 *   All other arguments, the workspace contract and the errors are those of
 *   tq_attend.
 */
int tq_attend_partial(const void* q, int q_dtype,
                      const uint8_t* packed_k, const uint16_t* norms_k,
                      const uint8_t* packed_v, const uint16_t* norms_v,
                      const int32_t* ctx_lens, int batch, int n_q_heads,
                      int gqa_ratio, int d, int bits_k, int bits_v, uint64_t seed,
                      int cap_tok, float sparse_v_thresh, int n_ctas,
                      void* workspace, size_t workspace_bytes, int* dev_status,
                      unsigned long long* sparse_v_skipped,
                      float* partial, void* stream);

/*
 * tq_attend_combine — merge the records of n_parts disjoint slices and
 * rotate the result back once:
 *   M = max_p m2_p, f_p = 2^(m2_p - M) (0 for an empty slice),
 *   l = sum_p f_p·l_p, acc = sum_p f_p·acc_p, out = D⊙(H·(acc / l)) / d.
 *   partials    float [n_parts][batch][n_q_heads][d + 2], 8-byte aligned
 *               (e.g. the all-gather of every device's tq_attend_partial
 *               output, in any order of the parts).
 *   n_parts >= 1; batch, n_q_heads >= 1; d = 64, 128 or 256.
 *   seed        the sign-vector seed of the cache.
 *   dev_status  device int, nullable: TQ_DEV_CTX_EMPTY when a (sequence,
 *               head) had no position in any slice (its output is 0).
 *   out         [batch][n_q_heads][d] of out_dtype, 16-byte aligned.
 * Errors: TQ_ERR_INVALID_ARG for a null or misaligned pointer or a bad
 * size or dtype; TQ_ERR_CUDA for a failed launch.
 */
int tq_attend_combine(const float* partials, int n_parts, int batch, int n_q_heads,
                      int d, uint64_t seed, int* dev_status, void* out, int out_dtype,
                      void* stream);

/*
 * Stage-2 residual sketch (QJL) and the unbiased inner-product estimate.
 * "We Built a Python Library That Cuts LLM Memory Usage by 80%", section
 * "Why not both stages?": the method has a second stage, a one-bit
 * correction of the stage-1 residual that makes inner products unbiased;
 * that page leaves it out of softmax attention because its variance hurts
 * there. The library therefore offers it for keys, as a score estimate, not
 * inside tq_attend. The page gives nothing more; the library's definition:
 *   r~    = R·x - nK·c[idx]/sqrt(d)   the key's stage-1 residual in rotated
 *                                      coordinates (= R·(x - x_hat)),
 *                                      R = H·diag(D)/sqrt(d), nK the stored
 *                                      fp16 norm, c the N(0,1) codebook
 *   S     d x d, i.i.d. N(0,1), supplied by the caller (one per model or
 *         layer; the same S for encode and scores)
 *   bit_i = 1 iff (S·r~)_i >= 0, i = 0..d-1, LSB-first, d/8 bytes per row
 *   gamma = ||r~||, fp16 round-to-nearest-even, saturated at 65504
 *   estimate <q, x> ~ <q~, nK·c[idx]/sqrt(d)> + gamma·sqrt(pi/2)/d·<S·q~, 2·bit - 1>
 * with q~ = R·q. For s ~ N(0, I), E[sign(s·r)(s·q)] = sqrt(2/pi)·<q, r>/|r|,
 * so the correction is unbiased for <q, x - x_hat> over the draw of S (up
 * to the fp16 rounding of gamma).
 *
 * tq_qjl_encode — sketch rows of n_tok keys of one sequence.
 *   k           [n_tok][n_kv_heads][d] fp16/bf16 keys (dtype), 16-byte aligned.
 *   projection  float [d][d], row i = projection vector i, 16-byte aligned.
 *   packed_k, norms_k  the keys' stage-1 cache (tq_encode's output for the
 *               same keys, seed and bits_k), rows tok_offset .. + n_tok - 1
 *               are read; packed_k 16-byte aligned.
 *   sketch      uint8 [n_kv_heads][cap_tok][d/8], rows tok_offset .. written.
 *   gamma       fp16 bits [n_kv_heads][cap_tok], same rows written.
 *   Other arguments as for tq_encode (bits_k 2..4); TQ_DEV_NORM_SATURATED
 *   reports a gamma above 65504.
 */
int tq_qjl_encode(const void* k, int dtype, int n_tok, int n_kv_heads, int d, int bits_k,
                  uint64_t seed, const float* projection, const uint8_t* packed_k,
                  const uint16_t* norms_k, uint8_t* sketch, uint16_t* gamma, int cap_tok,
                  int tok_offset, int* dev_status, void* stream);

/*
 * tq_qjl_scores — estimated attention scores estimate/sqrt(d) of every query
 * head against the first L_b = min(ctx_lens[b], cap_tok) cached keys:
 *   scores[b][h][t] = (<q~, nK_t·c[idx_t]/sqrt(d)>
 *                      + with_sketch·gamma_t·sqrt(pi/2)/d·<S·q~, 2·bit_t - 1>) / sqrt(d)
 * for t < L_b; entries t >= L_b are not written.
 *   q           [batch][n_q_heads][d] of q_dtype (TQ_F16 | TQ_BF16 | TQ_F32),
 *               16-byte aligned; kv head of query head h is h / gqa_ratio.
 *   packed_k, norms_k  stage-1 key cache [batch][n_kv_heads][cap_tok][...],
 *               packed_k 16-byte aligned.
 *   sketch, gamma  tq_qjl_encode's rows [batch][n_kv_heads][cap_tok][...],
 *               sketch 8-byte aligned; unused (may be NULL) when with_sketch = 0.
 *   projection  the S given to tq_qjl_encode; may be NULL when with_sketch = 0.
 *   with_sketch 1: the unbiased estimate; 0: the stage-1 score only.
 *   scores      float [batch][n_q_heads][cap_tok].
 *   ctx_lens, batch, n_q_heads, gqa_ratio (1..8), d, bits_k, seed, cap_tok,
 *   dev_status  as for tq_attend (ctx > cap_tok clamped with
 *               TQ_DEV_CTX_CLAMPED; ctx <= 0 writes nothing, TQ_DEV_CTX_EMPTY).
 */
int tq_qjl_scores(const void* q, int q_dtype, const uint8_t* packed_k, const uint16_t* norms_k,
                  const uint8_t* sketch, const uint16_t* gamma, const float* projection,
                  const int32_t* ctx_lens, int batch, int n_q_heads, int gqa_ratio, int d,
                  int bits_k, uint64_t seed, int cap_tok, int with_sketch, int* dev_status,
                  float* scores, void* stream);

/*
 * tq_attend_noalloc — tq_attend for callers that cannot allocate device
 * memory when they run attention (a fixed memory budget set at start-up, a
 * runtime that forbids allocations after initialization because they can
 * synchronize the device, or a plugin whose host owns every allocation).
 * None of the source pages has a counterpart; this is a library convenience.
 *
 * Same arguments and results as tq_attend, without workspace and
 * workspace_bytes: the scratch is one fixed 16 MiB device array inside the
 * library, created on each device together with the library's device code
 * and kept until the process exits. The call itself allocates and frees no
 * memory, with one exception on each device's first use:
 *   - Under CUDA's default lazy module loading, a device gets the library's
 *     device code, and with it the 16 MiB array, only when that code is
 *     first used there. The first tq_attend_noalloc call on a device looks
 *     up the array's address, which loads the module if nothing else has.
 *     Make that first call during initialization, before any stream capture
 *     (or set CUDA_MODULE_LOADING=EAGER, which creates the array with the
 *     CUDA context). Later calls reuse the address.
 *   - The address is kept for the life of the process: do not use this
 *     entry point on a device after cudaDeviceReset.
 *   - Limit: the problem's tq_attend_workspace_size must fit 16 MiB, i.e.
 *     batch · n_q_heads <= 54530 / 23887 / 8033 at d = 64 / 128 / 256;
 *     larger problems return TQ_ERR_UNSUPPORTED.
 *   - Every call on a device shares the array. Each call first clears the
 *     array's counter region on `stream`; calls whose execution overlaps on
 *     the GPU (other streams, other threads) race on it and give undefined
 *     results. Serialize them.
 */
int tq_attend_noalloc(const void* q, int q_dtype,
                      const uint8_t* packed_k, const uint16_t* norms_k,
                      const uint8_t* packed_v, const uint16_t* norms_v,
                      const int32_t* ctx_lens, int batch, int n_q_heads,
                      int gqa_ratio, int d, int bits_k, int bits_v, uint64_t seed,
                      int cap_tok, float sparse_v_thresh, int n_ctas,
                      int* dev_status, unsigned long long* sparse_v_skipped,
                      void* out, int out_dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
