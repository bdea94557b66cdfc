// engram_forward_no_alloc: the whole pass in a static device scratch array,
// for callers that cannot allocate device memory (a plugin given only its
// input and output buffers, a latency-critical loop where cudaMalloc/cudaFree
// would synchronise the device).  It adds an entry point and changes nothing
// in engram_forward, which it calls with the array as the workspace.
#include <mutex>

#include "engram_internal.cuh"

namespace {

constexpr size_t kScratchBytes = ENGRAM_NO_ALLOC_SCRATCH_BYTES;

// Held by every GPU that loads the library, until the process exits.
static __device__ __align__(256) unsigned char g_no_alloc_scratch[kScratchBytes];

// Device address of the array per device.  In host code the array's name is
// only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, looked up once per device with that device current.
std::mutex g_mu;
void* g_scratch_addr[256] = {};

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
    if (g_scratch_addr[dev] == nullptr) {
      void* addr = nullptr;
      e = cudaGetSymbolAddress(&addr, g_no_alloc_scratch);
      if (e != cudaSuccess || addr == nullptr)
        return engram::set_error(ENGRAM_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s",
                                 cudaGetErrorString(e));
      g_scratch_addr[dev] = addr;
    }
    scratch = g_scratch_addr[dev];
  }
  return engram_forward(cfg, weights, ids, B, T, hidden, y, state, scratch, kScratchBytes,
                        dev_status, stream);
}
