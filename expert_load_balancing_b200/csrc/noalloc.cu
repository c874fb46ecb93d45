// noalloc.cu -- the permutation entry point for callers that cannot allocate
// device memory (see kolibri_expert_permute_noalloc in kolibri_router.h).
//
// Its scratch lives in a fixed module-scope array.  Host code never passes
// the array's name to a kernel: in host code that name is only a stand-in.
// The device address is taken once per device with cudaGetSymbolAddress
// while that device is current, then reused.
#include <mutex>

#include "launch.h"
#include "common.cuh"

namespace kolibri {

namespace {

constexpr size_t kNoAllocScratchBytes = KOLIBRI_NOALLOC_SCRATCH_BYTES;  // held by every GPU that loads the library
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (resolved on the
// first call for that device).  Returns nullptr if the lookup fails.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();   // clear it, so no later launch check reports it as its own
      return nullptr;
    }
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
KOLIBRI_DEFINE_STATUS_TAKE(status_take_noalloc)

}  // namespace kolibri

using namespace kolibri;

extern "C" {

kolibri_status kolibri_expert_permute_noalloc(const int32_t* ids, int64_t N, int32_t E, int32_t K,
                                              int32_t* counts, int64_t* offsets, int32_t* perm,
                                              int32_t* inv, void* stream) {
  if (N < 1 || E < 1 || K < 1 || K >= E) return KOLIBRI_ERR_INVALID_ARG;
  if (E > KOLIBRI_MAX_EXPERTS || K > KOLIBRI_MAX_TOPK || (E % 4) != 0)
    return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (N * static_cast<int64_t>(K) >= (static_cast<int64_t>(1) << 31))
    return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (!ids || !counts || !offsets || !perm) return KOLIBRI_ERR_INVALID_ARG;
  // sizes whose scratch would not fit the fixed array are refused up front
  if (permute_layout(N, E, K).total > kNoAllocScratchBytes) return KOLIBRI_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = scratch_on_current_device();
  if (!scratch) return KOLIBRI_ERR_CUDA;
  // launch_permute clears what must start at zero (its ticket) on the stream
  const cudaError_t err = launch_permute(ids, N, E, K, counts, offsets, perm, inv, scratch,
                                         static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? KOLIBRI_OK : KOLIBRI_ERR_CUDA;
}

}  // extern "C"
