// tq_encode kernel: FP16 norm, randomized Hadamard rotation, Lloyd-Max
// index, LSB-first bit-packing — one pass over each K/V head vector.
//
// [TQAI §The Paper]: keep the norm in FP16, rotate the unit vector,
// quantize each coordinate with the precomputed Lloyd-Max codebook.
// [ADAPTQ §How it works, item 1]: y = (1/sqrt d)·H·D·x applied with a fast
// Walsh-Hadamard transform. [TQAI §What's Next]: indices bit-packed at
// 2/3/4 bits.
//
// Thread layout: four lanes per vector, 32 consecutive coordinates per lane
// (d = 128). A 256-thread block encodes 64 consecutive tokens of one kv head
// (K or V) per step, so its packed rows and norms form one contiguous range;
// blocks stride over the (tile, head, K/V) units. The kernel is bound by
// instruction issue, so the arithmetic uses two-wide fp32 operations:
//   load    4 x 16-byte loads per lane (the vector's 256 bytes, coalesced),
//           D applied by one XOR per fp16 pair
//   norm    16 paired FMAs + 2 shuffles
//   rotate  1 scalar + 4 paired butterfly stages, 2 cross-lane stages
//   index   zeta = z/n compared as z against n·t (symmetric half table),
//           counted with compare-and-set results
//   pack    the lane's 32 indices are 4·bits contiguous bytes of the row
#include "device_common.cuh"

namespace tq {
namespace {

constexpr int kEncThreads = 256;
constexpr int kEncTokens = kEncThreads / 4;

template <int BITS>
__device__ __forceinline__ void encode_vector(
    float (&x)[32], const Codebook& cb, int sub, unsigned gmask,
    uint8_t* row_dst, uint16_t* norm_dst, int* dev_status) {
  constexpr int kHalf = 1 << (BITS - 1);
  // ||x||^2 over the group of four lanes (pairs of coordinates per fma)
  float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float2 v = make_float2(x[2 * j], x[2 * j + 1]);
    ss2 = f2fma(v, v, ss2);
  }
  float ss = ss2.x + ss2.y;
  ss += __shfl_xor_sync(gmask, ss, 1);
  ss += __shfl_xor_sync(gmask, ss, 2);
  const float n = sqrtf(ss);

  // z = H·(D⊙x): coordinate 32·sub + i lives in register i of lane sub.
  // Stride 1 in scalar form, strides 2..16 on register pairs, strides 32 and
  // 64 across the four lanes (x' = partner + sign·x, sign = -1 on the upper
  // lane); every step rounds exactly like a scalar add or subtract.
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float u = x[2 * j], v = x[2 * j + 1];
    x[2 * j] = u + v;
    x[2 * j + 1] = u - v;
  }
#pragma unroll
  for (int s = 2; s < 32; s <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      if ((i & s) == 0) {
        const float2 u = make_float2(x[i], x[i + 1]), v = make_float2(x[i + s], x[i + s + 1]);
        const float2 p = f2add(u, v), m = f2sub(u, v);
        x[i] = p.x; x[i + 1] = p.y;
        x[i + s] = m.x; x[i + s + 1] = m.y;
      }
    }
  }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    const float sg = (sub & o) ? -1.f : 1.f;
    const float2 sg2 = make_float2(sg, sg);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float2 v = make_float2(x[2 * j], x[2 * j + 1]);
      const float2 p = make_float2(__shfl_xor_sync(gmask, v.x, o), __shfl_xor_sync(gmask, v.y, o));
      const float2 r = f2fma(v, sg2, p);
      x[2 * j] = r.x;
      x[2 * j + 1] = r.y;
    }
  }

  // idx = #{j : z/n >= t_j}, evaluated as z against n·t_j. Positive half of
  // the table: T_k = n·t_{half-1+k}, k = 1..half-1 (t_{half-1} = 0).
  // z >= 0: idx = half + #{k : T_k <= z};  z < 0: idx = half-1 - #{k : T_k < |z|}.
  // The strict comparison uses |z| lowered by one ulp. A zero vector keeps
  // n = 0, z = 0 and must land on idx = half: scale the table by 1 instead.
  // Counts are sums of compare results (0 or -1).
  const float sc = n > 0.f ? n : 1.f;
  float T[kHalf > 1 ? kHalf - 1 : 1];
#pragma unroll
  for (int k = 1; k < kHalf; ++k) T[k - 1] = sc * cb.threshold[kHalf - 1 + k];

  uint32_t words[BITS] = {};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float z = x[i];
    const bool neg = z < 0.f;
    const float a = __uint_as_float((__float_as_uint(z) & 0x7FFFFFFFu) - (neg ? 1u : 0u));
    uint32_t s = 0;                                   // = -count
#pragma unroll
    for (int k = 0; k < kHalf - 1; ++k) s += set_ge(a, T[k]);
    const uint32_t idx = neg ? (uint32_t)(kHalf - 1) + s : (uint32_t)kHalf - s;
    const int p = i * BITS, w = p >> 5, off = p & 31;
    words[w] += idx << off;                           // fields do not overlap
    if (off + BITS > 32) words[w + 1] += idx >> (32 - off);
  }

  if constexpr (BITS == 4) {
    *reinterpret_cast<uint4*>(row_dst + 16 * sub) =
        make_uint4(words[0], words[1], words[2], words[3]);
  } else if constexpr (BITS == 2) {
    *reinterpret_cast<uint2*>(row_dst + 8 * sub) = make_uint2(words[0], words[1]);
  } else {
    uint32_t* d32 = reinterpret_cast<uint32_t*>(row_dst + 12 * sub);
    d32[0] = words[0];
    d32[1] = words[1];
    d32[2] = words[2];
  }
  if (sub == 0) {
    *norm_dst = f32_to_f16_bits(fminf(n, 65504.f));
    if (n > 65504.f && dev_status) atomicOr(dev_status, TQ_DEV_NORM_SATURATED);
  }
}

// Grid-stride over (token tile, kv head, K/V): each group of four lanes
// encodes one vector per iteration; its half2 sign masks are built once.
__global__ void __launch_bounds__(kEncThreads)
encode_kernel(const __grid_constant__ EncodeArgs a,
              const __grid_constant__ Codebook cbk,
              const __grid_constant__ Codebook cbv,
              const __grid_constant__ SignMask sm) {
  // Programmatic dependent launch (a no-op without it): the next launch may
  // start; the input may come from the previous one, so wait before reading.
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;
  const unsigned gmask = 0xFu << (lane & ~3);
  // XOR masks that flip the fp16 sign bits of coordinates 2j (bit 15) and
  // 2j+1 (bit 31) of this lane's 16 half2 words where D = -1.
  uint32_t smask[16];
  {
    const uint32_t m = sm.w[sub];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      smask[j] = (((m >> (2 * j)) & 1u) << 15) | (((m >> (2 * j + 1)) & 1u) << 31);
  }
  const int tiles = (a.n_tok + kEncTokens - 1) / kEncTokens;
  const long long units = (long long)tiles * a.n_kv_heads * 2;
  for (long long u = blockIdx.x; u < units; u += gridDim.x) {
    const int tile = (int)(u % tiles);
    const int h = (int)((u / tiles) % a.n_kv_heads);
    const int is_v = (int)(u / ((long long)tiles * a.n_kv_heads));
    const int tok = tile * kEncTokens + (threadIdx.x >> 2);
    if (tok >= a.n_tok) continue;                     // whole groups of four

    const uint16_t* src = a.kv +
        ((size_t)(is_v * a.n_tok + tok) * a.n_kv_heads + h) * kHeadDim + 32 * sub;
    uint4 raw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) raw[k] = __ldcs(reinterpret_cast<const uint4*>(src) + k);
    float x[32];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t w4[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = unpack16x2(w4[j] ^ smask[4 * k + j], a.is_bf16);
        x[8 * k + 2 * j] = f.x;
        x[8 * k + 2 * j + 1] = f.y;
      }
    }

    const size_t row = (size_t)h * a.cap_tok + a.tok_offset + tok;
    const int bits = is_v ? a.bits_v : a.bits_k;
    const Codebook& cb = is_v ? cbv : cbk;
    uint8_t* packed = is_v ? a.packed_v : a.packed_k;
    uint16_t* norms = (is_v ? a.norms_v : a.norms_k) + row;
    const size_t rb = (size_t)kHeadDim * bits / 8;
    if (bits == 4)
      encode_vector<4>(x, cb, sub, gmask, packed + row * rb, norms, a.dev_status);
    else if (bits == 3)
      encode_vector<3>(x, cb, sub, gmask, packed + row * rb, norms, a.dev_status);
    else
      encode_vector<2>(x, cb, sub, gmask, packed + row * rb, norms, a.dev_status);
  }
}

}  // namespace

cudaError_t launch_encode(const EncodeArgs& a, const Codebook& cbk,
                          const Codebook& cbv, const SignMask& sm,
                          cudaStream_t stream) {
  // Enough resident blocks to cover every SM several times; each block then
  // strides over the (tile, head, K/V) units.
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sms = 148;
  }
  const long long units = (long long)((a.n_tok + kEncTokens - 1) / kEncTokens) * a.n_kv_heads * 2;
  const int grid = (int)(units < (long long)sms * 8 ? units : (long long)sms * 8);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kEncThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, encode_kernel, a, cbk, cbv, sm);
}

}  // namespace tq
