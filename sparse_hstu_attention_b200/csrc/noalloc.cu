// hstu_sla_fwd_noalloc: the SLA forward for callers that may not allocate
// device memory.  It runs exactly the hstu_sla_fwd path (work-list kernel +
// tcgen05 forward kernel), with the work lists and status word placed in a
// fixed-size array that lives in the library's own device memory instead of a
// caller-provided workspace.
#include <cuda.h>

#include <mutex>

#include "sla_common.cuh"

namespace {

// 2 MiB: the forward workspace of any batch with ceil(T/64) + B <= 131,040
// (about 8.3 million tokens).  Every GPU that loads the library keeps this
// array for the life of the process.
constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
// Per device: the context the address was looked up in and the address.  A
// device reset (or a release and re-creation of the primary context) makes
// a new context in which the array can sit elsewhere: the address is looked
// up again when the current context differs from the cached one.
struct ScratchEntry {
  unsigned long long ctx_id;
  void* addr;
};
ScratchEntry g_scratch[kMaxDevices];
std::mutex g_scratch_mutex;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Identifier of the context current on this thread (0 if the driver entry
// points are unavailable: the cache is then keyed by device alone).
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device.  In host code the
// symbol name is only a host-side handle; the device address must be looked up
// with that device current, once per device and context.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSTU_SLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HSTU_SLA_ERR_UNSUPPORTED;
  // binds the device's primary context to this thread (creating it after a
  // reset); allocates nothing
  if (cudaSetDevice(dev) != cudaSuccess) return HSTU_SLA_ERR_CUDA;
  const unsigned long long ctx = current_ctx_id();
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchEntry& e = g_scratch[dev];
  if (e.addr == nullptr || e.ctx_id != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return HSTU_SLA_ERR_CUDA;
    e.addr = p;
    e.ctx_id = ctx;
  }
  *out = e.addr;
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

extern "C" int hstu_sla_noalloc_get_error(hstu_stream_t stream) {
  void* scratch = nullptr;
  const int e = scratch_address(&scratch);
  if (e != HSTU_SLA_OK) return e;
  return hstu_sla_get_error(scratch, stream);
}
