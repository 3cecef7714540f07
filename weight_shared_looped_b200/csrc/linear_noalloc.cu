// tl_linear_noalloc: the quantised-weight linear layer (tl_linear) for callers
// that cannot allocate device memory while they run.
//
// Who needs it: a process whose device memory is reserved up front by another
// allocator (cudaMalloc can then fail, or stall the whole device because it
// synchronises), code that issues work while someone else's stream capture is
// open (an allocation made there is not part of the captured graph), and
// embedded or real-time callers with a fixed memory budget decided at start-up.
// tl_linear asks such a caller for a scratch buffer for its split-K partial
// sums; this variant uses a fixed buffer compiled into the library instead.
//
// The buffer is a file-scope __device__ array of kNoAllocScratchBytes (4 MiB).
// Every GPU that loads the library holds it until the process exits.  Calls
// whose partial sums need more than that are rejected before any launch.  All
// calls share the one buffer and it keeps the last call's contents; every call
// overwrites the part it reads, so nothing has to start at zero, but calls that
// overlap on the GPU (different streams, no ordering between them) race on it.
//
// Host code cannot hand the array's name to a kernel: on the host that name is
// a stand-in, not a device address.  The first call on each device looks up
// the array's device address with cudaGetSymbolAddress (with that device
// current) and keeps it; make that first call before any stream capture.
#include <cstring>
#include <mutex>

#include "tl_internal.cuh"

namespace tl {
namespace {

constexpr size_t kNoAllocScratchBytes = 4u << 20;
__device__ __align__(256) unsigned char g_linear_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

tl_status scratch_address(void** out) {
  int dev = -1;
  TL_CUDA(cudaGetDevice(&dev));
  TL_CHECK_ARG(dev >= 0 && dev < kMaxDevices, "device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_linear_scratch);
    if (e != cudaSuccess || p == nullptr)
      return set_error(TL_ERR_CUDA, "cudaGetSymbolAddress of the built-in scratch failed: %s",
                       cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return ok();
}

}  // namespace
}  // namespace tl

using namespace tl;

extern "C" __attribute__((visibility("default"))) tl_status tl_linear_noalloc(
    const uint32_t* packed, const uint16_t* scales, int N, int K, int group, const uint16_t* x,
    int T, float* y, tl_stream stream) {
  TL_TRY(check_linear(N, K, group, T));
  TL_CHECK_ARG(packed && scales && x && y, "NULL device pointer");
  const int S = linear_splits(N, K, T);
  const size_t need = S > 1 ? (size_t)S * T * N * sizeof(float) : 0;
  if (need > kNoAllocScratchBytes)
    return set_error(TL_ERR_INVALID_ARG,
                     "tl_linear_noalloc: N=%d K=%d T=%d needs %zu bytes of split-K scratch, above "
                     "the built-in %zu; use tl_linear with a caller buffer",
                     N, K, T, need, kNoAllocScratchBytes);
  TL_TRY(gemm_tc_init());
  void* scratch = nullptr;
  if (S > 1) TL_TRY(scratch_address(&scratch));
  return launch_linear(packed, scales, N, K, group, x, T, y, (float*)scratch,
                       (cudaStream_t)stream);
}
