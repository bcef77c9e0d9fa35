// permute_noalloc.cu -- moe_permute for callers that cannot allocate device memory.
//
// Some callers can't hand the library a workspace: a serving loop that
// reserves all device memory at start-up and forbids allocation afterwards,
// a plugin running inside another framework that owns every device
// allocation, or code that must not trigger the implicit device-wide
// synchronisation cudaMalloc/cudaFree can cause.  This entry point runs the
// same permutation kernels as moe_permute, with their scratch (the
// per-block expert histograms) in a fixed-size array compiled into the
// library instead of a caller-provided workspace.
#include <mutex>

#include "kernels.h"

namespace {

constexpr long long kNoallocMaxSlots = 131072;  // T * k
constexpr int kNoallocMaxExperts = 1024;
// Per-block histograms for the largest problem: one row of E counts per
// block of slots.  512 Ki int32 = 2 MiB, resident on every device that
// loads the library until the process exits.
constexpr size_t kScratchInts = 512u * 1024u;

static __device__ __align__(256) int32_t g_permute_scratch[kScratchInts];

constexpr int kMaxDevices = 128;
std::mutex g_mutex;
int32_t* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the host-side symbol is only a stand-in, never a device address).
moe_status_t scratch_address(int dev, int32_t** out) {
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_scratch_addr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_permute_noalloc(const int32_t* topk_ids, int T, int E, int k, int32_t* counts,
                                            int32_t* offsets, int32_t* sorted_token_ids, int32_t* inv_perm,
                                            void* stream) {
  if (!topk_ids || !counts || !offsets || !sorted_token_ids || !inv_perm) return MOE_ERR_INVALID_ARG;
  if (T < 1 || E < 1 || k < 1 || k > E || k > 64) return MOE_ERR_INVALID_ARG;
  const uintptr_t mis = (reinterpret_cast<uintptr_t>(topk_ids) | reinterpret_cast<uintptr_t>(counts) |
                         reinterpret_cast<uintptr_t>(offsets) | reinterpret_cast<uintptr_t>(sorted_token_ids) |
                         reinterpret_cast<uintptr_t>(inv_perm)) & 15u;
  if (mis) return MOE_ERR_ALIGNMENT;
  // Sizes beyond the built-in scratch are refused before anything is enqueued.
  if ((long long)T * k > kNoallocMaxSlots || E > kNoallocMaxExperts) return MOE_ERR_WORKSPACE;
  if ((size_t)moe::permute_num_blocks(T, k) * (size_t)E > kScratchInts) return MOE_ERR_WORKSPACE;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED_ARCH;
  int32_t* scratch = nullptr;
  const moe_status_t st = scratch_address(dev, &scratch);
  if (st != MOE_OK) return st;
  // Every histogram row the kernels read is written first in the same call,
  // so nothing has to be cleared; no device status word is kept here.
  const cudaError_t err = moe::launch_permute(topk_ids, T, E, k, counts, offsets, sorted_token_ids, inv_perm,
                                              scratch, nullptr, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
