// bl_noalloc.cu -- the absmean scale without a caller-provided workspace.
//
// The regular bitlinear_absmean needs a workspace for its per-chunk partial
// sums, which the caller allocates.  Some callers cannot allocate device
// memory when they need gamma: a host process whose device memory is owned by
// another runtime or memory pool that hands out no raw buffers, a service that
// reserves all of its device memory at start-up and forbids allocation later,
// or code on a latency path where cudaMalloc / cudaFree (which may synchronize
// the device) are not acceptable.  This entry point serves them: its scratch
// lives in a fixed device array that the library owns.
//
// The array is file-scope device memory: every GPU that loads the library
// holds kNoAllocScratchBytes of it until the process exits.  Host code cannot
// use the array's name as a device address, so the address is looked up once
// per device with cudaGetSymbolAddress and passed to the kernel.
#include <atomic>
#include <mutex>

#include "bitlinear.h"
#include "bl_common.cuh"
#include "bl_kernels.h"

namespace bl {
namespace {

// Header (the chunk counter) plus one fp64 partial per 8192-element chunk.
constexpr int64_t kNoAllocMaxChunks = 32768;
constexpr size_t kNoAllocScratchBytes = BL_WS_HEADER_BYTES + kNoAllocMaxChunks * sizeof(double);

static __device__ __align__(256) uint8_t g_absmean_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call per device).  Returns nullptr if the lookup fails.
void* scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_absmean_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace bl

extern "C" bl_status bitlinear_absmean_noalloc(const void* W, int wdt, int64_t N, int64_t K, float* gamma,
                                               void* stream) {
  if (W == nullptr || gamma == nullptr) return BL_ERR_INVALID_VALUE;
  if (!(wdt == BL_F32 || wdt == BL_BF16) || N < 1 || K < 1 || K > (int64_t{1} << 20)) return BL_ERR_INVALID_VALUE;
  if (N > (int64_t{1} << 32) / K) return BL_ERR_INVALID_VALUE;
  if (((reinterpret_cast<uintptr_t>(W) & 15) != 0) || ((reinterpret_cast<uintptr_t>(gamma) & 3) != 0))
    return BL_ERR_MISALIGNED;
  const int64_t chunks = (N * K + bl::kChunk - 1) / bl::kChunk;
  if (chunks > bl::kNoAllocMaxChunks) return BL_ERR_SCRATCH_LIMIT;
  void* scratch = bl::scratch_for_current_device();
  if (scratch == nullptr) return BL_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The chunk counter must start at zero; a previous call that did not finish
  // could have left it elsewhere.
  if (cudaMemsetAsync(scratch, 0, BL_WS_HEADER_BYTES, st) != cudaSuccess) return BL_ERR_CUDA;
  return bl::launch_absmean(W, wdt, N, K, scratch, gamma, st) == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}
