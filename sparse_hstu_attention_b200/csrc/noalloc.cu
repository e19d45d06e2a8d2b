// hstu_sla_fwd_noalloc: the SLA forward for callers that may not allocate
// device memory.  It runs exactly the hstu_sla_fwd path (work-list kernel +
// tcgen05 forward kernel), with the work lists and status word placed in a
// fixed-size array that lives in the library's own device memory instead of a
// caller-provided workspace.
#include <atomic>
#include <mutex>

#include "sla_common.cuh"

namespace {

// 2 MiB: the forward workspace of any batch with ceil(T/64) + B <= 131,040
// (about 8.3 million tokens).  Every GPU that loads the library keeps this
// array for the life of the process.
constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of g_noalloc_scratch on the current device.  In host code the
// symbol name is only a host-side handle; the device address must be looked up
// once per device, with that device current.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSTU_SLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HSTU_SLA_ERR_UNSUPPORTED;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    p = g_scratch_addr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return HSTU_SLA_ERR_CUDA;
      g_scratch_addr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return HSTU_SLA_OK;
}

}  // namespace

extern "C" int hstu_sla_fwd_noalloc(const hstu_sla_fwd_params* p, hstu_stream_t stream) {
  if (p == nullptr) return HSTU_SLA_ERR_INVALID_ARG;
  const size_t need = hstu_sla_workspace_bytes(HSTU_SLA_WS_FWD, p->total_tokens, p->B, p->H, p->d);
  if (need == 0) return HSTU_SLA_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return HSTU_SLA_ERR_WORKSPACE;  // batch too large
  void* scratch = nullptr;
  const int e = scratch_address(&scratch);
  if (e != HSTU_SLA_OK) return e;
  return hstu_sla_fwd(p, scratch, kNoAllocScratchBytes, stream);
}
