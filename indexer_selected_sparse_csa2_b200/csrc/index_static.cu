// csa_index_topk_noalloc: the decode indexer + Top-K without a caller
// workspace.
//
// Some callers cannot hand the library scratch memory: a serving runtime whose
// caching allocator already owns the whole GPU and gives out only the tensors
// it tracks, or a latency-critical loop that must not call cudaMalloc (which
// can synchronise the device and stall every other stream).  This entry point
// takes the same arguments as csa_index_topk minus the workspace and uses a
// fixed-size array in the library's device image instead.
//
// Properties a caller must know:
//   - The array holds kNoallocScratchBytes (16 MiB) on every GPU that loads
//     the library, for the life of the process.  Calls whose scratch need
//     (csa_index_workspace_size) exceeds it return CSA_ERR_WORKSPACE before
//     any launch.
//   - The first call on a device looks the array's device address up
//     (cudaGetSymbolAddress) with that device current and caches it; make
//     that first call before any stream capture.
//   - All calls on a device share the one array and it keeps the previous
//     call's contents; the kernels clear what must start at zero.  Calls that
//     can overlap on the GPU (different streams without ordering) race on it.
//   - No cudaMalloc, cudaFree or allocating library routine is called.
#include <mutex>

#include "select.cuh"

namespace csa {

constexpr size_t kNoallocScratchBytes = (size_t)16 << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

static std::mutex g_noalloc_mu;
static void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (cached per device).
static cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}

}  // namespace csa

using namespace csa;

extern "C" {

size_t csa_index_noalloc_capacity(void) { return kNoallocScratchBytes; }

csa_status csa_index_topk_noalloc(const csa_index_args* a, csa_stream_t stream) {
  // Argument checks are those of csa_index_topk: its workspace-size query
  // returns 0 for invalid arguments, and csa_index_topk reports why.
  if (!a) return CSA_ERR_INVALID_ARG;
  const size_t need = csa_index_workspace_size(a);
  if (need == 0) return csa_index_topk(a, nullptr, 0, stream);   // returns the argument error
  if (need > kNoallocScratchBytes) return CSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return CSA_ERR_CUDA;
  return csa_index_topk(a, scratch, kNoallocScratchBytes, stream);
}

}  // extern "C"
