// tq_encode kernel: FP16 norm, randomized Hadamard rotation, Lloyd-Max
// index, LSB-first bit-packing — one pass over each K/V head vector.
//
// Thread layout: d/32 lanes per vector (2, 4 or 8 for d = 64, 128, 256), 32
// consecutive coordinates per lane. A 256-thread block encodes 256/(d/32)
// consecutive tokens of one kv head (K or V) per step, so its packed rows and
// norms form one contiguous range; the grid is (tile blocks, kv head, K/V)
// and a block strides over its head's tiles. The per-vector arithmetic
// (encode_common.cuh) uses two-wide fp32 operations, since the kernel is
// bound by instruction issue:
//   load    4 x 16-byte loads per lane (the vector's 256 bytes, coalesced),
//           D applied by one XOR per fp16 pair
//   norm    16 paired FMAs + 2 shuffles
//   rotate  1 scalar + 4 paired butterfly stages, 2 cross-lane stages
//   index   zeta = z/n compared as |z| against n·t (symmetric half table)
//           by a binary search of saturated FMAs
//   pack    the lane's 32 indices are 4·bits contiguous bytes of the row
#include <atomic>
#include "encode_common.cuh"

namespace tq {
namespace {

constexpr int kEncThreads = 256;

// Grid (tile blocks, kv head, K/V): block (x, h, is_v) strides over the
// token tiles of one kv head's K or V; each group of d/32 lanes encodes one
// vector per iteration; its half2 sign masks are built once.
template <int D>
__global__ void __launch_bounds__(kEncThreads)
encode_kernel(const __grid_constant__ EncodeArgs a,
              const __grid_constant__ Codebook cbk,
              const __grid_constant__ Codebook cbv,
              const __grid_constant__ SignMask sm) {
  // Programmatic dependent launch (a no-op without it): the next launch may
  // start; the input may come from the previous one, so wait before reading.
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  constexpr int LPV = D / 32;                 // lanes per vector
  constexpr int kTokens = kEncThreads / LPV;  // tokens per tile
  const int lane = threadIdx.x & 31;
  const int sub = lane & (LPV - 1);
  const unsigned gmask = ((1u << LPV) - 1u) << (lane & ~(LPV - 1));
  uint32_t smask[16];
  sign_masks(sm, sub, smask);
  const int h = blockIdx.y;
  const int is_v = blockIdx.z;
  const int bits = is_v ? a.bits_v : a.bits_k;
  const Codebook& cb = is_v ? cbv : cbk;
  const size_t rb = (size_t)D * bits / 8;
  uint8_t* packed = (is_v ? a.packed_v : a.packed_k) + ((size_t)h * a.cap_tok + a.tok_offset) * rb;
  uint16_t* norms = (is_v ? a.norms_v : a.norms_k) + (size_t)h * a.cap_tok + a.tok_offset;
  const uint16_t* src0 = a.kv + ((size_t)is_v * a.n_tok * a.n_kv_heads + h) * D;
  const size_t tok_stride = (size_t)a.n_kv_heads * D;
  for (int tok = blockIdx.x * kTokens + threadIdx.x / LPV; tok < a.n_tok;
       tok += gridDim.x * kTokens) {
    // the destination row lies in the cache (bounds-checked build)
    if (!tq_check(a.tok_offset + tok < a.cap_tok, a.dev_status)) continue;
    float x[32];
    load_signed(src0 + tok * tok_stride, sub, a.is_bf16, smask, x);
    if (bits == 4)
      encode_vector<4, LPV>(x, cb, sub, gmask, packed + tok * rb, norms + tok, a.dev_status);
    else if (bits == 3)
      encode_vector<3, LPV>(x, cb, sub, gmask, packed + tok * rb, norms + tok, a.dev_status);
    else
      encode_vector<2, LPV>(x, cb, sub, gmask, packed + tok * rb, norms + tok, a.dev_status);
  }
}

template <int D>
cudaError_t launch_encode_d(const EncodeArgs& a, const Codebook& cbk, const Codebook& cbv,
                            const SignMask& sm, cudaStream_t stream) {
  // SM count of the current device, looked up once per device
  static std::atomic<int> cached[64] = {};
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
    if (!cached[dev]) {
      int n = 0;
      cached[dev] = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) ==
                            cudaSuccess && n > 0 ? n : 148;
    }
    sms = cached[dev];
  }
  // d = 128 with a few tiles of tokens: the tensor-core encode (the FWHT
  // kernel below when the driver's tensor-map call is unavailable)
  if (encode_tc_applies(a)) {
    const cudaError_t e = launch_encode_tc(a, cbk, cbv, sm, sms, stream);
    if (e != cudaErrorNotSupported) return e;
  }
  // grid.x: enough tile blocks that all (head, K/V) pairs cover every SM
  // about eight times; each block strides over its head's tiles
  constexpr int kTokens = kEncThreads / (D / 32);
  const int tiles = (a.n_tok + kTokens - 1) / kTokens;
  const int pairs = a.n_kv_heads * 2;
  int gx = (sms * 8 + pairs - 1) / pairs;
  if (gx > tiles) gx = tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gx, a.n_kv_heads, 2);
  cfg.blockDim = dim3(kEncThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, encode_kernel<D>, a, cbk, cbv, sm);
}

}  // namespace

cudaError_t launch_encode(const EncodeArgs& a, const Codebook& cbk,
                          const Codebook& cbv, const SignMask& sm,
                          cudaStream_t stream) {
  switch (a.d) {
    case 64: return launch_encode_d<64>(a, cbk, cbv, sm, stream);
    case 128: return launch_encode_d<128>(a, cbk, cbv, sm, stream);
    case 256: return launch_encode_d<256>(a, cbk, cbv, sm, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tq
