// tq_encode at d = 128 on the B200 tensor cores (tcgen05, TMEM, TMA).
//
// [ADAPTQ §How it works, item 1]: the rotation y = (1/sqrt d)·H·D·x. For a
// tile of 128 tokens of one kv head, z = H·(D⊙x) for every token is the
// product X·B of the tile X [128 tokens x 128 coordinates] with the
// constant B = diag(D)·H (H symmetric, entries +-1: exact in fp16 and
// bf16), accumulated in fp32. [TQAI §The Paper]: the norm in FP16, each
// coordinate quantized with the Lloyd-Max codebook; [TQAI §What's Next]:
// indices bit-packed.
//
// Roles (one persistent CTA per SM over the (K/V, kv head, tile) items):
//   warp 0       loads tiles with the tensor map (two 128 x 64 boxes,
//                128-byte swizzle) into a ring of kStages shared slots
//   warp 1       allocates tensor memory; one thread issues the eight
//                128 x 128 x 16 tcgen05.mma of a tile into one of kAcc fp32
//                accumulators (128 TMEM columns each) and commits them
//   warps 2..17  four epilogue groups of four warps; group g takes the
//                items j = g mod 4 of this CTA and accumulator g. Each
//                thread reads its token's row of the accumulator
//                (tcgen05.ld, 32 columns at a time): pass 1 sums z^2
//                (||x|| = ||z||/sqrt(d)), pass 2 takes the indices with the
//                FWHT encoder's arithmetic (quantize_pack) and stores the
//                packed row and the fp16 norm.
// Every wait is bounded (as in the attention kernel): a wait that gives up
// sets TQ_DEV_WAIT_TIMEOUT and its role stops; the producer then waits
// (bounded) for its loads still in flight, and the accumulators are freed
// after a CTA barrier.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "encode_common.cuh"
#include "tc_common.cuh"

namespace tq {
namespace {

constexpr int kTile = 128;                  // tokens per tile (MMA M)
constexpr int kDim = 128;                   // head dimension (MMA N and K)
constexpr int kStages = 4;                  // tiles in flight
constexpr int kAcc = 4;                     // TMEM accumulators = epilogue groups
constexpr int kWarps = 2 + 4 * kAcc;
constexpr int kThreads = 32 * kWarps;
constexpr int kTileBytes = kTile * kDim * 2;    // 32 KB (two 16 KB swizzled halves)
constexpr int kHalfBytes = kTileBytes / 2;
constexpr int kTmemCols = kAcc * kDim;          // 512
// shared memory: 1 KB alignment slack, kStages tiles, B, barriers, TMEM address
constexpr int kBarOff = kStages * kTileBytes + kTileBytes;
constexpr int kSmem = 1024 + kBarOff + 256;
constexpr long long kTcWaitLimit = 2000000000LL;    // cycles (~1 s)
static_assert(kTmemCols == 512, "one CTA per SM holds all 512 TMEM columns");
static_assert(kSmem <= 227 * 1024, "shared memory");

using tc::bar_arrive;
using tc::bar_expect;
using tc::bar_init;
using tc::saddr;
using tc::tmem_ld32;
using tc::umma_desc;
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) {
  return tc::bar_wait(bar, parity, kTcWaitLimit);
}
__host__ __device__ constexpr uint32_t umma_idesc(uint32_t fmt) {
  return tc::umma_idesc(fmt, kTile, kDim);
}

// Item j of the CTA's list -> (K/V, kv head, tile).
struct TcItem {
  int kv, h, t;
};
__device__ __forceinline__ TcItem tc_item(int item, int n_heads, int n_tiles) {
  TcItem it;
  it.t = item % n_tiles;
  it.h = (item / n_tiles) % n_heads;
  it.kv = item / (n_tiles * n_heads);
  return it;
}

template <int BITS>
__device__ __forceinline__ void epilogue_row(uint32_t tacc, const Codebook& cb, uint8_t* row,
                                             uint16_t* norm, bool valid, int* dev_status) {
  float z[32];
  // pass 1: ||z||^2 = d·||x||^2 (H·H = d·I); 64 columns per wait
  float2 ss = make_float2(0.f, 0.f), ss1 = ss;
#pragma unroll 1
  for (int c = 0; c < kDim / 64; ++c) {
    float zb[32];
    tc::tmem_ld32x2(tacc + 64 * c, tacc + 64 * c + 32, z, zb);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      ss = f2fma(make_float2(z[2 * j], z[2 * j + 1]), make_float2(z[2 * j], z[2 * j + 1]), ss);
      ss1 = f2fma(make_float2(zb[2 * j], zb[2 * j + 1]), make_float2(zb[2 * j], zb[2 * j + 1]), ss1);
    }
  }
  ss = f2add(ss, ss1);
  const float n = sqrtf((ss.x + ss.y) * (1.f / kDim));
  // pass 2: indices of 32 coordinates at a time, BITS words each
#pragma unroll 1
  for (int c = 0; c < kDim / 32; ++c) {
    tmem_ld32(tacc + 32 * c, z);
    uint32_t w[BITS];
    quantize_pack<BITS>(z, n, cb, w);
    if (valid) {
      if constexpr (BITS == 4) {
        *reinterpret_cast<uint4*>(row + 16 * c) = make_uint4(w[0], w[1], w[2], w[3]);
      } else if constexpr (BITS == 2) {
        *reinterpret_cast<uint2*>(row + 8 * c) = make_uint2(w[0], w[1]);
      } else {
        uint32_t* d32 = reinterpret_cast<uint32_t*>(row + 12 * c);
        d32[0] = w[0];
        d32[1] = w[1];
        d32[2] = w[2];
      }
    }
  }
  if (valid) {
    *norm = f32_to_f16_bits(fminf(n, 65504.f));
    if (n > 65504.f && dev_status) atomicOr(dev_status, TQ_DEV_NORM_SATURATED);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
encode_tc_kernel(const __grid_constant__ EncodeArgs a, const __grid_constant__ CUtensorMap tmap,
                 const __grid_constant__ Codebook cbk, const __grid_constant__ Codebook cbv,
                 const __grid_constant__ SignMask sm) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = saddr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;                 // 1 KB aligned
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sX = base;                                     // kStages tiles
  const uint32_t sB = base + kStages * kTileBytes;              // the constant B
  const uint32_t bars = base + kBarOff;
  auto full_bar = [&](int s) { return bars + 8 * s; };
  auto empty_bar = [&](int s) { return bars + 8 * (kStages + s); };
  auto accfull_bar = [&](int g) { return bars + 8 * (2 * kStages + g); };
  auto accfree_bar = [&](int g) { return bars + 8 * (2 * kStages + kAcc + g); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + 8 * (2 * kStages + 2 * kAcc));
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  // ---- B = diag(D)·H as 128 rows (output coordinate n) of 128 K-elements
  // (input coordinate k), K-major, 128-byte swizzle: 16-byte chunk j of the
  // 128-byte row n of half h sits at chunk j ^ (n & 7).
  {
    const uint16_t one = a.is_bf16 ? 0x3F80u : 0x3C00u;        // +1 in bf16 / fp16
    for (int c = tid; c < kDim * 16; c += kThreads) {
      const int n = c >> 4, kc = c & 15, h = kc >> 3, j = kc & 7;
      uint32_t wv[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        uint32_t pair = 0;
#pragma unroll
        for (int f = 0; f < 2; ++f) {
          const int k = 8 * kc + e + f;
          const uint32_t neg = ((sm.w[k >> 5] >> (k & 31)) & 1u) ^ (__popc(k & n) & 1u);
          pair |= (uint32_t)(one | (neg << 15)) << (16 * f);
        }
        wv[e >> 1] = pair;
      }
      *reinterpret_cast<uint4*>(smem + kStages * kTileBytes + h * kHalfBytes + n * 128 +
                                ((j ^ (n & 7)) << 4)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      bar_init(full_bar(s), 1);
      bar_init(empty_bar(s), 1);
    }
    for (int g = 0; g < kAcc; ++g) {
      bar_init(accfull_bar(g), 1);
      bar_init(accfree_bar(g), 4);              // one arrive per epilogue warp
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  // the generic-proxy writes of B become visible to the tensor core's proxy
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
                 ::"r"(saddr(tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  const int n_tiles = (a.n_tok + kTile - 1) / kTile;
  const int n_items = 2 * a.n_kv_heads * n_tiles;
  const int my_items = n_items > (int)blockIdx.x
                           ? (n_items - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                           : 0;
  auto item_of = [&](int j) { return tc_item((int)blockIdx.x + j * (int)gridDim.x, a.n_kv_heads, n_tiles); };

  // The inputs may come from the previous launch in the stream.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");

  if (warp == 0) {
    // ---- producer: two 128 x 64 boxes per tile (coordinates: element in
    // the vector, kv head, token row of the [K; V] stack)
    if (lane == 0) {
      const uint64_t tm = reinterpret_cast<uint64_t>(&tmap);
      int j = 0;
      for (; j < my_items; ++j) {
        const int s = j % kStages;
        if (*reinterpret_cast<volatile int*>(abort_flag) ||
            !bar_wait(empty_bar(s), ((j / kStages) & 1) ^ 1)) {
          atomicExch(abort_flag, 1);
          break;
        }
        const TcItem it = item_of(j);
        const int row = it.kv * a.n_tok + it.t * kTile;
        bar_expect(full_bar(s), kTileBytes);
        for (int hf = 0; hf < 2; ++hf)
          asm volatile(
              "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
              " [%0], [%1, {%2, %3, %4}], [%5];\n"
              ::"r"(sX + s * kTileBytes + hf * kHalfBytes), "l"(tm), "r"(64 * hf), "r"(it.h),
                "r"(row), "r"(full_bar(s)) : "memory");
      }
      // loads still in flight complete before the CTA can end
      for (int k = j > kStages ? j - kStages : 0; k < j; ++k)
        bar_wait(full_bar(k % kStages), (k / kStages) & 1);
    }
  } else if (warp == 1) {
    // ---- MMA issue: accumulator g = j mod kAcc
    if (lane == 0) {
      const uint32_t idesc = umma_idesc(a.is_bf16 ? 1u : 0u);
      int j = 0;
      for (; j < my_items; ++j) {
        const int s = j % kStages, g = j % kAcc;
        if (*reinterpret_cast<volatile int*>(abort_flag) ||
            !bar_wait(full_bar(s), (j / kStages) & 1) ||
            !bar_wait(accfree_bar(g), ((j / kAcc) & 1) ^ 1)) {
          atomicExch(abort_flag, 1);
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
        const uint32_t d_tmem = tmem + g * kDim;
#pragma unroll
        for (int kk = 0; kk < kDim / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          const uint64_t ad = umma_desc(sX + s * kTileBytes + off);
          const uint64_t bd = umma_desc(sB + off);
          asm volatile(
              "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
              " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
              ::"r"(d_tmem), "l"(ad), "l"(bd), "r"(idesc), "r"(kk) : "memory");
        }
        // the tile's slot is free, and the accumulator full, once they complete
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n"
                     ::"r"(empty_bar(s)) : "memory");
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n"
                     ::"r"(accfull_bar(g)) : "memory");
      }
      if (j > 0) bar_wait(accfull_bar((j - 1) % kAcc), ((j - 1) / kAcc) & 1);   // last MMAs done
    }
  } else {
    // ---- epilogue group g: items j = g, g + kAcc, ...; thread = token row
    const int g = (warp - 2) >> 2;
    const int quad = warp & 3;                 // TMEM lanes this warp may access
    const int r = 32 * quad + lane;            // token row of the tile
    for (int j = g; j < my_items; j += kAcc) {
      const bool ok = bar_wait(accfull_bar(g), (j / kAcc) & 1);
      if (!__all_sync(0xFFFFFFFFu, ok) || *reinterpret_cast<volatile int*>(abort_flag)) {
        if (lane == 0) atomicExch(abort_flag, 1);
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
      const TcItem it = item_of(j);
      const int tok = it.t * kTile + r;
      // (and, in the bounds-checked build, its row lies in the cache)
      const bool valid = tok < a.n_tok && tq_check(a.tok_offset + tok < a.cap_tok, a.dev_status);
      const int bits = it.kv ? a.bits_v : a.bits_k;
      const size_t rb = (size_t)kDim * bits / 8;
      const size_t rowi = (size_t)it.h * a.cap_tok + a.tok_offset + (valid ? tok : 0);
      uint8_t* row = (it.kv ? a.packed_v : a.packed_k) + rowi * rb;
      uint16_t* norm = (it.kv ? a.norms_v : a.norms_k) + rowi;
      const Codebook& cb = it.kv ? cbv : cbk;
      const uint32_t tacc = tmem + ((uint32_t)(32 * quad) << 16) + g * kDim;
      if (bits == 4)
        epilogue_row<4>(tacc, cb, row, norm, valid, a.dev_status);
      else if (bits == 3)
        epilogue_row<3>(tacc, cb, row, norm, valid, a.dev_status);
      else
        epilogue_row<2>(tacc, cb, row, norm, valid, a.dev_status);
      asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
      __syncwarp();
      if (lane == 0) bar_arrive(accfree_bar(g));
    }
  }
  if (tid == 0 && *reinterpret_cast<volatile int*>(abort_flag) && a.dev_status)
    atomicOr(a.dev_status, TQ_DEV_WAIT_TIMEOUT);

  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n"
                 ::"r"(tmem), "r"(kTmemCols) : "memory");
}

// cuTensorMapEncodeTiled, looked up once through the runtime (the library
// does not link the driver library directly).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  static std::mutex mu;
  EncodeTiledFn f = fn.load();
  if (f) return f;
  std::lock_guard<std::mutex> lock(mu);
  if (!fn.load()) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn.store(reinterpret_cast<EncodeTiledFn>(p));
  }
  return fn.load();
}

}  // namespace

// Whether the tensor-core path takes this call: d = 128, at least a few
// tiles of tokens (small calls, such as one token, keep the FWHT kernel).
bool encode_tc_applies(const EncodeArgs& a) {
  return a.d == kDim && a.n_tok >= 4 * kTile && a.n_kv_heads <= 65535;
}

cudaError_t launch_encode_tc(const EncodeArgs& a, const Codebook& cbk, const Codebook& cbv,
                             const SignMask& sm, int sms, cudaStream_t stream) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  // the input [2][n_tok][n_kv_heads][d] as a 3-D tensor: (element, kv head,
  // token row of the K block followed by the V block)
  CUtensorMap tm;
  const cuuint64_t dims[3] = {(cuuint64_t)kDim, (cuuint64_t)a.n_kv_heads,
                              (cuuint64_t)a.n_tok * 2};
  const cuuint64_t strides[2] = {(cuuint64_t)kDim * 2, (cuuint64_t)a.n_kv_heads * kDim * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)kTile};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (enc(&tm, a.is_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
          const_cast<uint16_t*>(a.kv), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  static std::atomic<bool> configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(encode_tc_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  const int n_tiles = (a.n_tok + kTile - 1) / kTile;
  const int n_items = 2 * a.n_kv_heads * n_tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_items < sms ? n_items : sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, encode_tc_kernel, a, tm, cbk, cbv, sm);
}

}  // namespace tq
