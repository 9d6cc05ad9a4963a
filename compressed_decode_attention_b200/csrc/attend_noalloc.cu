// tq_attend_noalloc: tq_attend without a caller-supplied workspace.
//
// Some callers cannot allocate device memory at the point where they run
// attention: code that has a fixed device-memory budget decided at start-up,
// runtimes that forbid allocation after initialization (an allocation can
// synchronize the device and stall other streams), and plugins embedded in a
// host application that owns all device allocations. For them this entry
// point takes its scratch from one fixed array compiled into the library.
//
// The array is created on a device together with the library's device code.
// Under CUDA's default lazy module loading that happens on the first use of
// that code on the device, which for a caller of this entry point alone is
// the address lookup of its first call: that first call can allocate (the
// module and the array) and belongs in initialization, outside any stream
// capture. The array is kept until the process exits and is shared by every
// call on that device. Its size caps the problem: batch · n_q_heads <= 54530
// / 23887 / 8033 at d = 64 / 128 / 256 (see kNoAllocScratchBytes).
#include <mutex>

#include "tq.h"
#include "tq_internal.h"

namespace tq {
namespace {

// 16 MiB: partial-result slots (d + 2 floats per query head) for up to 1024
// CTAs plus the counters and the per-(batch, query head) slots.
constexpr size_t kNoAllocScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device. The name of a
// __device__ array in host code only stands in for it; the address has to be
// queried once per device with that device current. It is kept for the life
// of the process, so the entry point must not be used on a device after
// cudaDeviceReset (which unloads the module and frees the array).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace tq

extern "C" int tq_attend_noalloc(
    const void* q, int q_dtype, const uint8_t* packed_k, const uint16_t* norms_k,
    const uint8_t* packed_v, const uint16_t* norms_v, const int32_t* ctx_lens,
    int batch, int n_q_heads, int gqa_ratio, int d, int bits_k, int bits_v,
    uint64_t seed, int cap_tok, float sparse_v_thresh, int n_ctas, int* dev_status,
    unsigned long long* sparse_v_skipped, void* out, int out_dtype, void* stream) {
  using namespace tq;
  const size_t need = tq_attend_workspace_size(batch, n_q_heads, cap_tok, d);
  if (need == 0) return TQ_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return TQ_ERR_UNSUPPORTED;   // beyond the fixed scratch
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return TQ_ERR_CUDA;
  // The counters must start at zero; clear them on the caller's stream so a
  // previous call that did not finish cleanly cannot leave stale counts.
  if (cudaMemsetAsync(scratch, 0, attend_counter_bytes(batch, n_q_heads),
                      (cudaStream_t)stream) != cudaSuccess)
    return TQ_ERR_CUDA;
  return tq_attend(q, q_dtype, packed_k, norms_k, packed_v, norms_v, ctx_lens, batch,
                   n_q_heads, gqa_ratio, d, bits_k, bits_v, seed, cap_tok,
                   sparse_v_thresh, n_ctas, scratch, kNoAllocScratchBytes, dev_status,
                   sparse_v_skipped, out, out_dtype, stream);
}
