// engram_forward_no_alloc: the whole pass in a static device scratch array,
// for callers that cannot allocate device memory (a plugin given only its
// input and output buffers, a latency-critical loop where cudaMalloc/cudaFree
// would synchronise the device).  It adds an entry point and changes nothing
// in engram_forward, which it calls with the array as the workspace.
#include <cuda.h>

#include <mutex>

#include "engram_internal.cuh"

namespace {

constexpr size_t kScratchBytes = ENGRAM_NO_ALLOC_SCRATCH_BYTES;

// Held by every GPU that loads the library, until the process exits.
static __device__ __align__(256) unsigned char g_no_alloc_scratch[kScratchBytes];

// Device address of the array per device.  In host code the array's name is
// only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, looked up with that device current.  The address
// belongs to the device's current context: after cudaDeviceReset (or any
// other teardown of the primary context) the module is loaded again and the
// array may move.  So each cached address is tagged with the unique id of
// the context it was looked up in (cuCtxGetId; ids are never reused within a
// process) and looked up again when the current context's id differs.
struct Cached {
  unsigned long long ctx_id = 0;
  void* addr = nullptr;
};
std::mutex g_mu;
Cached g_scratch[256];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context; false when there is no
// current context yet or the driver offers no context ids.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool resolved = false;
  if (!resolved) {  // (under g_mu)
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    cudaGetLastError();
    resolved = true;
  }
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

}  // namespace

extern "C" engram_status engram_forward_no_alloc(const engram_config* cfg,
                                                 const engram_weights* weights, const int64_t* ids,
                                                 int32_t B, int32_t T, const void* hidden, void* y,
                                                 const engram_state* state, uint32_t* dev_status,
                                                 engram_stream stream) {
  size_t need = 0;
  engram_status st = engram_forward_workspace_size(cfg, B, T, &need);
  if (st != ENGRAM_OK) return st;
  if (need > kScratchBytes)
    return engram::set_error(ENGRAM_ERR_INVALID_ARG,
                             "engram_forward_no_alloc: B=%d T=%d needs %zu bytes of scratch but the "
                             "static scratch holds %zu; split the batch",
                             B, T, need, kScratchBytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return engram::set_error(ENGRAM_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 256)
    return engram::set_error(ENGRAM_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    unsigned long long ctx = 0;
    const bool have_ctx = current_context_id(&ctx);
    Cached& c = g_scratch[dev];
    if (!have_ctx || c.addr == nullptr || c.ctx_id != ctx) {
      void* addr = nullptr;
      e = cudaGetSymbolAddress(&addr, g_no_alloc_scratch);
      if (e != cudaSuccess || addr == nullptr)
        return engram::set_error(ENGRAM_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s",
                                 cudaGetErrorString(e));
      // the lookup made the primary context current if it was not yet
      c.addr = addr;
      c.ctx_id = current_context_id(&ctx) ? ctx : 0;
      if (c.ctx_id == 0) c.addr = nullptr;   // no context ids: look up again next call
      scratch = addr;
    } else {
      scratch = c.addr;
    }
  }
  return engram_forward(cfg, weights, ids, B, T, hidden, y, state, scratch, kScratchBytes,
                        dev_status, stream);
}
